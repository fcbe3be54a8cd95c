// moe_prefill.cu -- the prefill path: route, bucket the (token, expert) pairs per expert, then
// grouped gate/up and down over the buckets.
//
// Bucketing (histogram -> exclusive scan -> stable scatter) groups the T*k pairs by expert with
// ascending token order inside each expert, so every expert's tokens are contiguous and each
// expert's weights are read once per layer however many tokens it serves (the pages "Qwen-tin"
// and "--moe-direct-io" note that a long prompt touches nearly every expert of a layer).
// The grouped gate/up and down GEMMs over the buckets run on the tensor cores (tcgen05, see
// moe_prefill_tc.cu): gate/up writes h = SiLU(g) * u in bf16, down adds w * y into an fp32
// output accumulator with red.add, and a last kernel converts the accumulator to bf16.
#include "moe_internal.cuh"

namespace moe {

moe_status_t launch_route(const uint16_t *x, const float *wr, const float *bias, int T, int H, int E, int k,
                          int32_t *idx_out, float *w_out, cudaStream_t st);
moe_status_t launch_route_tc(const uint16_t *x, const float *wr, const float *bias, int T, int H, int E, int k,
                             int32_t *idx_out, float *w_out, uint16_t *planes, float *lg, uint32_t *status,
                             cudaStream_t st);
moe_status_t launch_tc_prefill_gemms(const uint8_t *packed, int T, int H, int I, int E, int k, const int32_t *counts,
                                     const int32_t *offsets, int32_t *nt_start, int4 *ntab, const int32_t *pair_tok,
                                     const float *pair_w, float *pscale, const uint16_t *x, uint16_t *x16,
                                     int32_t *xexp, uint16_t *h16, int8_t *hexp, float *out_acc, uint32_t *status,
                                     cudaStream_t st);

namespace {

// ------------------------------------------------------------------------------ bucketing
__global__ void bucket_hist_kernel(const int32_t *idx, int T, int k, int E, int32_t *blockhist) {
    extern __shared__ int hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int t0 = blockIdx.x * kScatterTokens;
    const int t1 = min(T, t0 + kScatterTokens);
    for (int p = t0 * k + threadIdx.x; p < t1 * k; p += blockDim.x) atomicAdd(&hist[idx[p]], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) blockhist[(size_t)blockIdx.x * E + e] = hist[e];
}

// counts[e], offsets[e] (exclusive scan, offsets[E] = T*k) and, in place, blockhist[b][e] ->
// first output position of block b's pairs of expert e. One CTA of 1024 threads; each expert's
// token blocks are split over tpe = 1024 / E threads (rounded down to a power of two), so that
// the per-expert walks over the blocks are tpe times shorter.
__global__ void bucket_scan_kernel(int32_t *blockhist, int nblk, int E, int32_t *counts, int32_t *offsets) {
    __shared__ int warp_tot[32];
    __shared__ int part[1024];      // part[e * tpe + q]: pairs of expert e in thread q's blocks
    __shared__ int excl_e[kMaxE];
    int tpe = 1;
    while (tpe * 2 * E <= 1024) tpe *= 2;
    const int tid = threadIdx.x, ex = tid / tpe, q = tid - ex * tpe;
    const int b0 = (int)((long long)nblk * q / tpe), b1 = (int)((long long)nblk * (q + 1) / tpe);
    int mine = 0;
    if (ex < E)
        for (int b = b0; b < b1; ++b) mine += blockhist[(size_t)b * E + ex];
    part[tid] = mine;
    __syncthreads();
    // block-wide exclusive scan of the experts' totals (thread e holds expert e's)
    const int e = tid, lane = tid & 31, w = tid >> 5;
    int c = 0;
    if (e < E)
        for (int j = 0; j < tpe; ++j) c += part[e * tpe + j];
    int incl = c;
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_tot[w] = incl;
    __syncthreads();
    if (w == 0) {
        int v = warp_tot[lane];
        int iv = v;
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, iv, off);
            if (lane >= off) iv += o;
        }
        warp_tot[lane] = iv - v;
    }
    __syncthreads();
    if (e < E) {
        const int excl = warp_tot[w] + incl - c;
        counts[e] = c;
        offsets[e] = excl;
        if (e == E - 1) offsets[E] = excl + c;
        excl_e[e] = excl;
    }
    __syncthreads();
    if (ex < E) {
        int run = excl_e[ex];
        for (int j = 0; j < q; ++j) run += part[ex * tpe + j];
        for (int b = b0; b < b1; ++b) {
            const int h = blockhist[(size_t)b * E + ex];
            blockhist[(size_t)b * E + ex] = run;
            run += h;
        }
    }
}

// One CTA of 256 threads per token block: its pairs in rounds of 256 (warp w of a round takes
// pairs 32w .. 32w+31 of it), ranked inside the warp by match_any and across the round's warps by
// a per-expert prefix in shared memory, so the order inside each expert's bucket is ascending
// (token, slot). Shared memory: cur[E] (next free position of each expert), cnt[8][E].
constexpr int kScatterThreads = 256;
__global__ void __launch_bounds__(kScatterThreads) bucket_scatter_kernel(const int32_t *idx, const float *w, int T,
                                                                         int k, int E, const int32_t *blockbase,
                                                                         int32_t *pair_tok, float *pair_w) {
    extern __shared__ int sm[];
    int *cur = sm;
    int *cnt = sm + E;
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    for (int e = threadIdx.x; e < E; e += kScatterThreads) cur[e] = blockbase[(size_t)blockIdx.x * E + e];
    const int t0 = blockIdx.x * kScatterTokens;
    const int p0 = t0 * k, p1 = min(T, t0 + kScatterTokens) * k;
    for (int base = p0; base < p1; base += kScatterThreads) {
        for (int i = threadIdx.x; i < 8 * E; i += kScatterThreads) cnt[i] = 0;
        __syncthreads();
        const int p = base + threadIdx.x;
        const bool ok = p < p1;
        const int e = ok ? idx[p] : -1 - lane;
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        if (ok && rank == 0) cnt[wp * E + e] = __popc(peers);
        __syncthreads();
        for (int ee = threadIdx.x; ee < E; ee += kScatterThreads) {
            int run = cur[ee];
            for (int j = 0; j < 8; ++j) {
                const int c = cnt[j * E + ee];
                cnt[j * E + ee] = run;
                run += c;
            }
            cur[ee] = run;
        }
        __syncthreads();
        if (ok) {
            const int pos = cnt[wp * E + e] + rank;
            pair_tok[pos] = p / k;
            pair_w[pos] = w[p];
        }
        __syncthreads();
    }
}

// out = bf16(acc), four elements per thread and step (n a multiple of 4)
__global__ void convert_kernel(const float4 *acc, uint2 *out, size_t n4) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        const float4 v = acc[i];
        const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
        out[i] = make_uint2(*reinterpret_cast<const uint32_t *>(&a), *reinterpret_cast<const uint32_t *>(&b));
    }
}

}  // namespace

// Routing and bucketing: idx / w of every (token, slot) pair, the experts' counts and offsets and
// the pair lists (token, weight) in bucket order, all in the workspace.
moe_status_t launch_prefill_route(const uint16_t *x, const float *wr, const float *bias, int T, int H, int I, int E,
                                  int k, int32_t *idx_out, float *w_out, void *ws, cudaStream_t st) {
    const PrefillWs L = prefill_ws_layout(T, H, I, E, k);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    int32_t *idx = reinterpret_cast<int32_t *>(w8 + L.idx);
    float *wt = reinterpret_cast<float *>(w8 + L.w);
    int32_t *counts = reinterpret_cast<int32_t *>(w8 + L.counts);
    int32_t *offsets = reinterpret_cast<int32_t *>(w8 + L.offsets);
    int32_t *bh = reinterpret_cast<int32_t *>(w8 + L.blockhist);
    int32_t *ptok = reinterpret_cast<int32_t *>(w8 + L.pair_tok);
    float *pw = reinterpret_cast<float *>(w8 + L.pair_w);
    const size_t P = (size_t)T * k;
    moe_status_t s = launch_route_tc(x, wr, bias, T, H, E, k, idx, wt, reinterpret_cast<uint16_t *>(w8 + L.planes),
                                     reinterpret_cast<float *>(w8 + L.lg), &reinterpret_cast<Control *>(w8)->status, st);
    if (s != MOE_OK) return s;
    if (idx_out && cudaMemcpyAsync(idx_out, idx, P * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (w_out && cudaMemcpyAsync(w_out, wt, P * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return MOE_ERR_CUDA;
    bucket_hist_kernel<<<L.nblk, 256, E * sizeof(int), st>>>(idx, T, k, E, bh);
    bucket_scan_kernel<<<1, 1024, 0, st>>>(bh, L.nblk, E, counts, offsets);
    bucket_scatter_kernel<<<L.nblk, kScatterThreads, 9 * E * sizeof(int), st>>>(idx, wt, T, k, E, bh, ptok, pw);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// The expert GEMMs over the buckets that launch_prefill_route left in the workspace, and the
// conversion of the fp32 accumulator to bf16.
moe_status_t launch_prefill_experts(const uint16_t *x, const void *packed, int T, int H, int I, int E, int k,
                                    uint16_t *out, void *ws, cudaStream_t st) {
    const PrefillWs L = prefill_ws_layout(T, H, I, E, k);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    float *oacc = reinterpret_cast<float *>(w8 + L.out_acc);
    if (cudaMemsetAsync(oacc, 0, (size_t)T * H * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
    moe_status_t s = launch_tc_prefill_gemms(
        static_cast<const uint8_t *>(packed), T, H, I, E, k, reinterpret_cast<const int32_t *>(w8 + L.counts),
        reinterpret_cast<const int32_t *>(w8 + L.offsets), reinterpret_cast<int32_t *>(w8 + L.nt_start),
        reinterpret_cast<int4 *>(w8 + L.ntab), reinterpret_cast<const int32_t *>(w8 + L.pair_tok),
        reinterpret_cast<const float *>(w8 + L.pair_w), reinterpret_cast<float *>(w8 + L.pscale), x,
        reinterpret_cast<uint16_t *>(w8 + L.x16), reinterpret_cast<int32_t *>(w8 + L.xexp),
        reinterpret_cast<uint16_t *>(w8 + L.h), reinterpret_cast<int8_t *>(w8 + L.hexp), oacc,
        &reinterpret_cast<Control *>(w8)->status, st);
    if (s != MOE_OK) return s;
    const size_t n4 = (size_t)T * H / 4;
    const DeviceInfo *dev = device_info();
    if (dev == nullptr) return MOE_ERR_CUDA;
    const size_t nb = (n4 + 255) / 256 < (size_t)dev->sms * 8 ? (n4 + 255) / 256 : (size_t)dev->sms * 8;
    convert_kernel<<<(unsigned)nb, 256, 0, st>>>(reinterpret_cast<const float4 *>(oacc), reinterpret_cast<uint2 *>(out), n4);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t launch_prefill(const uint16_t *x, const float *wr, const float *bias, const void *packed, int T, int H,
                            int I, int E, int k, uint16_t *out, int32_t *idx_out, float *w_out, void *ws,
                            cudaStream_t st) {
    const moe_status_t s = launch_prefill_route(x, wr, bias, T, H, I, E, k, idx_out, w_out, ws, st);
    if (s != MOE_OK) return s;
    return launch_prefill_experts(x, packed, T, H, I, E, k, out, ws, st);
}

}  // namespace moe
