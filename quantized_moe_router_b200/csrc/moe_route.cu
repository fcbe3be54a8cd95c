// moe_route.cu -- router logits + top-k + softmax renormalisation for any number of tokens.
//
// One CTA per 32 tokens computes all E logits l = x W_r^T (+ bias) of its tokens into shared
// memory, then one warp per token runs the top-k + softmax of moe_topk.cuh over them. The logits
// are an fp32 GEMM: for each chunk of 256 experts the CTA walks H in 32-wide slices staged in
// shared memory (x widened from bf16, exact; the next slice is fetched into registers while the
// current one is multiplied), every thread accumulating 4 tokens x 8 experts with packed fp32x2
// FMAs (fp32 products and sums, as the routing step requires). Each CTA reads the router weights
// once from L2 per 32 tokens.
#include "moe_internal.cuh"
#include "moe_topk.cuh"

namespace moe {
namespace {

constexpr int kRT = 32;    // tokens per CTA
constexpr int kRE = 256;   // experts per chunk
constexpr int kRK = 32;    // K slice
constexpr int kRThreads = 256;

// Thread (ty = warp, tx = lane) owns tokens 4 ty .. 4 ty + 3 and experts 4 tx .. 4 tx + 3 and
// 128 + 4 tx .. 128 + 4 tx + 3 of the chunk (so that a warp's W reads are two contiguous 512-byte
// rows of the slice). Shared memory: logits [kRT][E] | x slice [kRK][kRT] | W slice [kRK][kRE].
__global__ void __launch_bounds__(kRThreads) route_kernel(const uint16_t *__restrict__ x, const float *__restrict__ wr,
                                                          const float *__restrict__ bias, int T, int H, int E, int k,
                                                          int32_t *idx_out, float *w_out) {
    extern __shared__ __align__(16) float rsm[];
    float *lg = rsm;                                  // [kRT][E]
    float *xs = rsm + (size_t)kRT * E;                // [kRK][kRT]
    float *ws = xs + kRK * kRT;                       // [kRK][kRE]
    const int tid = threadIdx.x, tx = tid & 31, ty = tid >> 5;
    const int t0 = blockIdx.x * kRT;
    const int nt = min(kRT, T - t0);
    grid_dep_wait();
    for (int e0 = 0; e0 < E; e0 += kRE) {
        float2 acc[4][4];   // token i, experts (2j, 2j+1)
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = make_float2(0.f, 0.f);
        // the next slice is loaded into registers while the current one is multiplied
        const int xr = tid >> 2, xc = (tid & 3) * 8;
        const int e = e0 + tid;
        uint4 xv_next = make_uint4(0, 0, 0, 0);
        float4 wv_next[kRK / 4];
        auto load_slice = [&](int k0) {
            if (tid < 128 && xr < nt) xv_next = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)(t0 + xr) * H + k0 + xc));
            const float4 *src = reinterpret_cast<const float4 *>(wr + (size_t)e * H + k0);
#pragma unroll
            for (int q = 0; q < kRK / 4; ++q) wv_next[q] = (e < E) ? __ldg(src + q) : make_float4(0.f, 0.f, 0.f, 0.f);
        };
        load_slice(0);
        for (int k0 = 0; k0 < H; k0 += kRK) {
            // x slice: 32 tokens x 32 values (threads 0..127, 8 bf16 each); W slice: 256 experts x 32
            if (tid < 128) {
                const uint32_t w[4] = {xv_next.x, xv_next.y, xv_next.z, xv_next.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    xs[(xc + 2 * q) * kRT + xr] = __uint_as_float(w[q] << 16);
                    xs[(xc + 2 * q + 1) * kRT + xr] = __uint_as_float(w[q] & 0xFFFF0000u);
                }
            }
#pragma unroll
            for (int q = 0; q < kRK / 4; ++q) {
                ws[(4 * q + 0) * kRE + tid] = wv_next[q].x;
                ws[(4 * q + 1) * kRE + tid] = wv_next[q].y;
                ws[(4 * q + 2) * kRE + tid] = wv_next[q].z;
                ws[(4 * q + 3) * kRE + tid] = wv_next[q].w;
            }
            __syncthreads();
            if (k0 + kRK < H) load_slice(k0 + kRK);
#pragma unroll 4
            for (int kk = 0; kk < kRK; ++kk) {
                const float4 xv = *reinterpret_cast<const float4 *>(xs + kk * kRT + 4 * ty);
                const float4 w0 = *reinterpret_cast<const float4 *>(ws + kk * kRE + 4 * tx);
                const float4 w1 = *reinterpret_cast<const float4 *>(ws + kk * kRE + 128 + 4 * tx);
                const float xa[4] = {xv.x, xv.y, xv.z, xv.w};
                const float2 wp[4] = {make_float2(w0.x, w0.y), make_float2(w0.z, w0.w), make_float2(w1.x, w1.y),
                                      make_float2(w1.z, w1.w)};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 xx = make_float2(xa[i], xa[i]);
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = __ffma2_rn(xx, wp[j], acc[i][j]);
                }
            }
            __syncthreads();
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int ee = e0 + (j < 4 ? 4 * tx + j : 128 + 4 * tx + (j - 4));
                const float v = (j & 1) ? acc[i][j >> 1].y : acc[i][j >> 1].x;
                if (ee < E) lg[(4 * ty + i) * E + ee] = v + (bias ? __ldg(bias + ee) : 0.f);
            }
    }
    __syncthreads();
    for (int i = ty; i < nt; i += kRThreads / 32) {
        int idx;
        float w;
        warp_topk_softmax(lg + (size_t)i * E, false, E, k, tx, idx, w);
        if (tx < k) {
            idx_out[(size_t)(t0 + i) * k + tx] = idx;
            w_out[(size_t)(t0 + i) * k + tx] = w;
        }
    }
}

}  // namespace

moe_status_t launch_route(const uint16_t *x, const float *wr, const float *bias, int T, int H, int E, int k,
                          int32_t *idx_out, float *w_out, cudaStream_t st) {
    const DeviceInfo *dev = device_info();
    if (!dev) return MOE_ERR_CUDA;
    const size_t smem = ((size_t)kRT * E + (size_t)kRK * kRT + (size_t)kRK * kRE) * sizeof(float);
    if ((int)smem > dev->max_smem_optin) return MOE_ERR_UNSUPPORTED;
    static bool attr_set[64] = {false};
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64) return MOE_ERR_CUDA;
    if (!attr_set[d]) {
        if (cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dev->max_smem_optin) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
        attr_set[d] = true;
    }
    const unsigned blocks = (unsigned)((T + kRT - 1) / kRT);
    route_kernel<<<blocks, kRThreads, smem, st>>>(x, wr, bias, T, H, E, k, idx_out, w_out);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
