// moe_route.cu -- router logits + top-k + softmax renormalisation for any number of tokens.
//
// One CTA handles kRouteTokens tokens: each warp computes the fp32 logits of a strided set of
// experts for all of the CTA's tokens (so each router row is read once per CTA and each x row
// comes from L1), the logits land in shared memory, and one warp per token runs the top-k.
#include "moe_internal.cuh"
#include "moe_topk.cuh"

namespace moe {
namespace {

constexpr int kRouteTokens = 8;
constexpr int kRouteWarps = 8;

__global__ void __launch_bounds__(kRouteWarps * 32) route_kernel(const uint16_t *__restrict__ x,
                                                                 const float *__restrict__ wr,
                                                                 const float *__restrict__ bias, int T,
                                                                 int H, int E, int k, int32_t *idx_out,
                                                                 float *w_out) {
    extern __shared__ __align__(16) float lg[];  // [kRouteTokens][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * kRouteTokens;
    const int nt = min(kRouteTokens, T - t0);
    grid_dep_wait();
    for (int e = warp; e < E; e += kRouteWarps) {
        const float *wrow = wr + (size_t)e * H;
        float acc[kRouteTokens];
#pragma unroll
        for (int i = 0; i < kRouteTokens; ++i) acc[i] = 0.f;
        for (int h = lane * 8; h < H; h += 256) {
            const float4 w0 = __ldg(reinterpret_cast<const float4 *>(wrow + h));
            const float4 w1 = __ldg(reinterpret_cast<const float4 *>(wrow + h + 4));
#pragma unroll
            for (int i = 0; i < kRouteTokens; ++i) {
                if (i < nt) {
                    const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)(t0 + i) * H + h));
                    float a = acc[i];
                    a += w0.x * __uint_as_float(xv.x << 16) + w0.y * __uint_as_float(xv.x & 0xFFFF0000u);
                    a += w0.z * __uint_as_float(xv.y << 16) + w0.w * __uint_as_float(xv.y & 0xFFFF0000u);
                    a += w1.x * __uint_as_float(xv.z << 16) + w1.y * __uint_as_float(xv.z & 0xFFFF0000u);
                    a += w1.z * __uint_as_float(xv.w << 16) + w1.w * __uint_as_float(xv.w & 0xFFFF0000u);
                    acc[i] = a;
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kRouteTokens; ++i) {
            float a = acc[i];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
            if (lane == 0 && i < nt) lg[i * E + e] = a + (bias ? bias[e] : 0.f);
        }
    }
    __syncthreads();
    for (int i = warp; i < nt; i += kRouteWarps) {
        int idx;
        float w;
        warp_topk_softmax(lg + i * E, false, E, k, lane, idx, w);
        if (lane < k) {
            idx_out[(size_t)(t0 + i) * k + lane] = idx;
            w_out[(size_t)(t0 + i) * k + lane] = w;
        }
    }
}

}  // namespace

moe_status_t launch_route(const uint16_t *x, const float *wr, const float *bias, int T, int H, int E, int k,
                          int32_t *idx_out, float *w_out, cudaStream_t st) {
    const size_t smem = (size_t)kRouteTokens * E * sizeof(float);
    const unsigned blocks = (unsigned)((T + kRouteTokens - 1) / kRouteTokens);
    route_kernel<<<blocks, kRouteWarps * 32, smem, st>>>(x, wr, bias, T, H, E, k, idx_out, w_out);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
