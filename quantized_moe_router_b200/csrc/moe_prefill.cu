// moe_prefill.cu -- the prefill path: route, bucket the (token, expert) pairs per expert, then
// grouped gate/up and down over the buckets.
//
// Bucketing (histogram -> exclusive scan -> stable scatter) groups the T*k pairs by expert with
// ascending token order inside each expert, so every expert's tokens are contiguous and each
// expert's weights are read once per layer however many tokens it serves (the pages "Qwen-tin"
// and "--moe-direct-io" note that a long prompt touches nearly every expert of a layer).
// Grouped gate/up: one CTA per (expert, 8-row block); the block's packed tiles are brought in
// with one bulk copy and the 8 warps split the expert's tokens (8 per MMA n-tile). Its
// epilogue applies SiLU-GLU and writes h (bf16 hi + lo) and the per-group sums of h.
// Grouped down: one CTA per (expert, 16-row block); the epilogue adds w * y into the fp32
// output accumulator with red.add. A last kernel converts the accumulator to bf16.
#include "moe_internal.cuh"

namespace moe {

moe_status_t launch_route(const uint16_t *x, const float *wr, const float *bias, int T, int H, int E, int k,
                          int32_t *idx_out, float *w_out, cudaStream_t st);

namespace {

constexpr int kPW = 8;  // warps per grouped-GEMM CTA

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
// first output position of block b's pairs of expert e.
__global__ void bucket_scan_kernel(int32_t *blockhist, int nblk, int E, int32_t *counts, int32_t *offsets) {
    __shared__ int warp_tot[32];
    const int e = threadIdx.x;  // blockDim.x = 1024 >= E
    int c = 0;
    if (e < E)
        for (int b = 0; b < nblk; ++b) c += blockhist[(size_t)b * E + e];
    // block-wide exclusive scan of c
    const int lane = e & 31, w = e >> 5;
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
    const int excl = warp_tot[w] + incl - c;
    if (e < E) {
        counts[e] = c;
        offsets[e] = excl;
        if (e == E - 1) offsets[E] = excl + c;
        int run = excl;
        for (int b = 0; b < nblk; ++b) {
            const int h = blockhist[(size_t)b * E + e];
            blockhist[(size_t)b * E + e] = run;
            run += h;
        }
    }
}

// One warp per token block: pairs in ascending (token, slot) order, so the order inside each
// expert's bucket is ascending token.
__global__ void bucket_scatter_kernel(const int32_t *idx, const float *w, int T, int k, int E,
                                      const int32_t *blockbase, int32_t *pair_tok, float *pair_w) {
    extern __shared__ int cur[];
    const int lane = threadIdx.x;
    for (int e = lane; e < E; e += 32) cur[e] = blockbase[(size_t)blockIdx.x * E + e];
    __syncwarp();
    const int t0 = blockIdx.x * kScatterTokens;
    const int t1 = min(T, t0 + kScatterTokens);
    for (int base = t0 * k; base < t1 * k; base += 32) {
        const int p = base + lane;
        const bool ok = p < t1 * k;
        const int e = ok ? idx[p] : -1 - lane;
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        if (ok) {
            const int pos = cur[e] + rank;
            pair_tok[pos] = p / k;
            pair_w[pos] = w[p];
        }
        __syncwarp();
        if (ok && rank == 0) cur[e] += __popc(peers);
        __syncwarp();
    }
}

// ------------------------------------------------------------------------------ grouped GEMMs
struct GroupArgs {
    const uint16_t *x;
    const uint8_t *packed;
    int T, H, I, E, k;
    const int32_t *counts, *offsets, *pair_tok;
    const float *pair_w;
    const float *xsum;
    uint16_t *h_hi, *h_lo;
    float *hsum, *out_acc;
    uint64_t wait_ns;
    uint32_t *status;
};

template <int BITS, bool GU>
__device__ void grouped_tiles(const GroupArgs &a, const uint8_t *tiles, int ntiles, int rb, int e) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int n_e = a.counts[e], base = a.offsets[e];
    const int NT = (n_e + 7) >> 3;
    const int TB = tile_bytes(BITS);
    const int GI = a.I / kGroup;
    for (int nt = warp; nt < NT; nt += kPW) {
        const int q = nt * 8 + g, q0 = nt * 8 + 2 * t, q1 = q0 + 1;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int kg = 0; kg < ntiles; ++kg) {
            const uint8_t *tile = tiles + (size_t)kg * TB;
            const uint4 lo = *reinterpret_cast<const uint4 *>(tile + 16 * lane);
            uint4 hi8 = make_uint4(0, 0, 0, 0);
            uint2 hi6 = make_uint2(0, 0);
            if (BITS == 8) hi8 = *reinterpret_cast<const uint4 *>(tile + kLoBytes + 16 * lane);
            if (BITS == 6) hi6 = *reinterpret_cast<const uint2 *>(tile + kLoBytes + 8 * lane);
            const uint2 sz = *reinterpret_cast<const uint2 *>(tile + kLoBytes + hi_bytes(BITS) + 8 * g);
            const float sA = half_lo(sz.x), zA = half_hi(sz.x), sB = half_lo(sz.y), zB = half_hi(sz.y);
            uint32_t b[8] = {0, 0, 0, 0, 0, 0, 0, 0}, b2[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            float X0 = 0.f, X1 = 0.f;
            if (GU) {
                if (q < n_e) {
                    const uint4 *xp = reinterpret_cast<const uint4 *>(a.x + (size_t)a.pair_tok[base + q] * a.H +
                                                                      kg * kGroup + 16 * t);
                    const uint4 xa = __ldg(xp), xb = __ldg(xp + 1);
                    b[0] = xa.x; b[1] = xa.y; b[2] = xa.z; b[3] = xa.w;
                    b[4] = xb.x; b[5] = xb.y; b[6] = xb.z; b[7] = xb.w;
                }
                if (q0 < n_e) X0 = a.xsum[(size_t)a.pair_tok[base + q0] * (a.H / kGroup) + kg];
                if (q1 < n_e) X1 = a.xsum[(size_t)a.pair_tok[base + q1] * (a.H / kGroup) + kg];
                tile_group_mma<BITS>(lo, hi8, hi6, b, nullptr, sA, zA, sB, zB, X0, X1, acc);
            } else {
                if (q < n_e) {
                    const size_t off = (size_t)(base + q) * a.I + kg * kGroup + 16 * t;
                    const uint4 *hp = reinterpret_cast<const uint4 *>(a.h_hi + off);
                    const uint4 *lp = reinterpret_cast<const uint4 *>(a.h_lo + off);
                    const uint4 ha = __ldcg(hp), hb = __ldcg(hp + 1), la = __ldcg(lp), lb = __ldcg(lp + 1);
                    b[0] = ha.x; b[1] = ha.y; b[2] = ha.z; b[3] = ha.w;
                    b[4] = hb.x; b[5] = hb.y; b[6] = hb.z; b[7] = hb.w;
                    b2[0] = la.x; b2[1] = la.y; b2[2] = la.z; b2[3] = la.w;
                    b2[4] = lb.x; b2[5] = lb.y; b2[6] = lb.z; b2[7] = lb.w;
                }
                if (q0 < n_e) X0 = __ldcg(a.hsum + (size_t)(base + q0) * GI + kg);
                if (q1 < n_e) X1 = __ldcg(a.hsum + (size_t)(base + q1) * GI + kg);
                tile_group_mma<BITS>(lo, hi8, hi6, b, b2, sA, zA, sB, zB, X0, X1, acc);
            }
        }
        for (int col = 0; col < 2; ++col) {
            const int qq = nt * 8 + 2 * t + col;
            const bool valid = qq < n_e;
            if (GU) {
                const float gate = acc[col], up = acc[2 + col];
                const float h = gate / (1.f + expf(-gate)) * up;
                const __nv_bfloat16 hi = __float2bfloat16_rn(h);
                const __nv_bfloat16 lo = __float2bfloat16_rn(h - __bfloat162float(hi));
                float part = 0.f;
                if (valid) {
                    const size_t o = (size_t)(base + qq) * a.I + rb * 8 + g;
                    a.h_hi[o] = __bfloat16_as_ushort(hi);
                    a.h_lo[o] = __bfloat16_as_ushort(lo);
                    part = __bfloat162float(hi) + __bfloat162float(lo);
                }
                part += __shfl_xor_sync(0xffffffffu, part, 4);
                part += __shfl_xor_sync(0xffffffffu, part, 8);
                part += __shfl_xor_sync(0xffffffffu, part, 16);
                if (g == 0 && valid) red_add_f32(a.hsum + (size_t)(base + qq) * GI + (rb >> 3), part);
            } else if (valid) {
                const int tok = a.pair_tok[base + qq];
                const float wgt = a.pair_w[base + qq];
                const int row = rb * 16 + g;
                red_add_f32(a.out_acc + (size_t)tok * a.H + row, wgt * acc[col]);
                red_add_f32(a.out_acc + (size_t)tok * a.H + row + 8, wgt * acc[2 + col]);
            }
        }
    }
}

template <bool GU>
__global__ void __launch_bounds__(kPW * 32) grouped_kernel(const GroupArgs a) {
    extern __shared__ __align__(128) uint8_t tiles[];
    __shared__ __align__(8) uint64_t bar;
    const int e = blockIdx.x, rb = blockIdx.y;
    if (a.counts[e] == 0) return;
    const PackedExpert pe = reinterpret_cast<const PackedExpert *>(a.packed + sizeof(PackedHeader))[e];
    const int TB = tile_bytes(pe.bits);
    const int G = a.H / kGroup, GI = a.I / kGroup;
    const int ntiles = GU ? G : GI;
    const uint8_t *src = a.packed + pe.offset +
                         (GU ? (size_t)rb * G * TB : gu_tiles(a.H, a.I) * TB + (size_t)rb * GI * TB);
    const uint32_t mb = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(mb, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t bytes = (uint32_t)(ntiles * TB);
        mbar_expect_tx(mb, bytes);
        bulk_g2s(smem_u32(tiles), src, bytes, mb);
    }
    if (!mbar_wait(mb, 0, a.wait_ns, a.status)) return;
    if (pe.bits == 4)
        grouped_tiles<4, GU>(a, tiles, ntiles, rb, e);
    else if (pe.bits == 6)
        grouped_tiles<6, GU>(a, tiles, ntiles, rb, e);
    else
        grouped_tiles<8, GU>(a, tiles, ntiles, rb, e);
}

// per-token sums of x over each 64-column group (sequential fp32 sum, as in the decode kernel)
__global__ void xsum_kernel(const uint16_t *x, int T, int H, float *xsum) {
    const int G = H / kGroup;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < (size_t)T * G; i += (size_t)gridDim.x * blockDim.x) {
        const uint16_t *xp = x + (i / G) * H + (i % G) * kGroup;
        float s = 0.f;
        for (int j = 0; j < kGroup; ++j) s += bf16_bits_to_float(xp[j]);
        xsum[i] = s;
    }
}

__global__ void convert_kernel(const float *acc, uint16_t *out, size_t n) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[i]));
}

}  // namespace

size_t prefill_max_tiles_bytes(int H, int I) {
    const int G = H / kGroup, GI = I / kGroup;
    return (size_t)(G > GI ? G : GI) * tile_bytes(8);
}

moe_status_t launch_prefill(const uint16_t *x, const float *wr, const float *bias, const void *packed, int T, int H,
                            int I, int E, int k, uint16_t *out, int32_t *idx_out, float *w_out, void *ws,
                            cudaStream_t st) {
    const PrefillWs L = prefill_ws_layout(T, H, I, E, k);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    int32_t *idx = reinterpret_cast<int32_t *>(w8 + L.idx);
    float *wt = reinterpret_cast<float *>(w8 + L.w);
    int32_t *counts = reinterpret_cast<int32_t *>(w8 + L.counts);
    int32_t *offsets = reinterpret_cast<int32_t *>(w8 + L.offsets);
    int32_t *bh = reinterpret_cast<int32_t *>(w8 + L.blockhist);
    int32_t *ptok = reinterpret_cast<int32_t *>(w8 + L.pair_tok);
    float *pw = reinterpret_cast<float *>(w8 + L.pair_w);
    float *hsum = reinterpret_cast<float *>(w8 + L.hsum);
    float *oacc = reinterpret_cast<float *>(w8 + L.out_acc);
    const size_t P = (size_t)T * k;
    moe_status_t s = launch_route(x, wr, bias, T, H, E, k, idx, wt, st);
    if (s != MOE_OK) return s;
    if (idx_out && cudaMemcpyAsync(idx_out, idx, P * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (w_out && cudaMemcpyAsync(w_out, wt, P * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(hsum, 0, P * (I / kGroup) * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(oacc, 0, (size_t)T * H * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
    float *xs = reinterpret_cast<float *>(w8 + L.xsum);
    {
        const size_t nx = (size_t)T * (H / kGroup);
        xsum_kernel<<<(unsigned)((nx + 255) / 256 < 2048 ? (nx + 255) / 256 : 2048), 256, 0, st>>>(x, T, H, xs);
    }
    bucket_hist_kernel<<<L.nblk, 256, E * sizeof(int), st>>>(idx, T, k, E, bh);
    bucket_scan_kernel<<<1, 1024, 0, st>>>(bh, L.nblk, E, counts, offsets);
    bucket_scatter_kernel<<<L.nblk, 32, E * sizeof(int), st>>>(idx, wt, T, k, E, bh, ptok, pw);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;

    GroupArgs a;
    a.x = x; a.packed = static_cast<const uint8_t *>(packed);
    a.T = T; a.H = H; a.I = I; a.E = E; a.k = k;
    a.counts = counts; a.offsets = offsets; a.pair_tok = ptok; a.pair_w = pw; a.xsum = xs;
    a.h_hi = reinterpret_cast<uint16_t *>(w8 + L.h_hi);
    a.h_lo = reinterpret_cast<uint16_t *>(w8 + L.h_lo);
    a.hsum = hsum; a.out_acc = oacc;
    a.wait_ns = wait_limit_ns();
    a.status = &reinterpret_cast<Control *>(w8)->status;
    const size_t smem = prefill_max_tiles_bytes(H, I);
    const DeviceInfo *dev = device_info();
    if ((int)smem + 1024 > dev->max_smem_optin) return MOE_ERR_UNSUPPORTED;
    static bool attr_set[16] = {false};
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) return MOE_ERR_CUDA;
    if (d < 16 && !attr_set[d]) {
        if (cudaFuncSetAttribute(grouped_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dev->max_smem_optin - 1024) != cudaSuccess ||
            cudaFuncSetAttribute(grouped_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dev->max_smem_optin - 1024) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_set[d] = true;
    }
    grouped_kernel<true><<<dim3(E, I / 8), kPW * 32, smem, st>>>(a);
    grouped_kernel<false><<<dim3(E, H / 16), kPW * 32, smem, st>>>(a);
    const size_t n = (size_t)T * H;
    convert_kernel<<<(unsigned)((n + 1023) / 1024 < 4096 ? (n + 1023) / 1024 : 4096), 256, 0, st>>>(oacc, out, n);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
