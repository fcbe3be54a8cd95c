// moe_route_tc.cu -- router logits of the prefill path on the 5th-generation tensor cores.
//
// Routing needs the fp32 logits l = x W_r^T (+ bias) of every token, a dense contraction of
// T x H by E x H (4.3 GFLOP for 4096 tokens, 256 experts, H = 2048). x is bf16; the router rows
// are fp32. Every fp32 value is the exact sum of three bf16 values,
//     w = w1 + w2 + w3,  w1 = bf16(w), w2 = bf16(w - w1), w3 = bf16(w - w1 - w2)
// (each remainder is exact in fp32 and the last one has at most 8 significant bits), so
//     x w = x w1 + x w2 + x w3
// with every product exact in fp32. One kernel splits W_r into the three bf16 planes; the logits
// kernel then runs bf16 x bf16 tcgen05 MMAs into an fp32 TMEM accumulator, the three planes against
// the same x tile at every K step, and a third kernel takes the top-k + softmax of each token's
// logits (moe_topk.cuh). The logits differ from an fp32 dot product only by the order of the
// additions.
// Logits kernel: one CTA per 128 tokens x 64 experts; one thread brings the x tile (128 rows x 64
// columns) and the three plane tiles (64 rows x 64 columns) of each K step with 2-D tensor copies
// into a 4-stage ring, one thread issues the MMAs (12 per K step, M = 128, N = 64, K = 16) and
// frees each stage with tcgen05.commit, and 4 epilogue warps read the accumulator (one token per
// thread), add the bias and store the fp32 logits. Every wait is bounded.
#include <mutex>

#include "moe_tc.cuh"
#include "moe_topk.cuh"

namespace moe {
namespace {

constexpr int kRM = 128;                             // tokens per CTA (UMMA M)
constexpr int kRN = 64;                              // experts per CTA (UMMA N)
constexpr int kRStages = 4;
constexpr int kRPlanes = 3;
constexpr int kRABytes = kRM * 128;                  // x tile: 128 rows x 64 bf16
constexpr int kRBBytes = kRN * 128;                  // one plane's router tile: 64 rows x 64 bf16
constexpr int kRStageBytes = kRABytes + kRPlanes * kRBBytes;
constexpr int kRThreads = 6 * 32;                    // copies, MMA, 4 epilogue warps
constexpr int kRSmem = kRStages * kRStageBytes + 1024;

struct RouteTcShared {
    uint64_t full[kRStages];
    uint64_t empty[kRStages];
    uint64_t acc, fin;
    uint32_t tmem;
    volatile int abort;
};

// w -> its three bf16 planes (planes [3][E x H], plane i at i * n)
__global__ void router_split_kernel(const float4 *__restrict__ wr, size_t n4, uint2 *__restrict__ planes) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        const float4 v = wr[i];
        const float w[4] = {v.x, v.y, v.z, v.w};
        uint32_t p[3][2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint16_t b[3][2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float x = w[2 * h + j];
                const __nv_bfloat16 b1 = __float2bfloat16_rn(x);
                const float r1 = x - __bfloat162float(b1);
                const __nv_bfloat16 b2 = __float2bfloat16_rn(r1);
                const float r2 = r1 - __bfloat162float(b2);
                const __nv_bfloat16 b3 = __float2bfloat16_rn(r2);
                b[0][j] = __bfloat16_as_ushort(b1);
                b[1][j] = __bfloat16_as_ushort(b2);
                b[2][j] = __bfloat16_as_ushort(b3);
            }
#pragma unroll
            for (int q = 0; q < 3; ++q) p[q][h] = (uint32_t)b[q][0] | ((uint32_t)b[q][1] << 16);
        }
#pragma unroll
        for (int q = 0; q < 3; ++q) planes[q * n4 + i] = make_uint2(p[q][0], p[q][1]);
    }
}

__device__ __forceinline__ bool rt_wait(RouteTcShared &S, uint64_t *bar, uint32_t parity, uint64_t limit,
                                        uint32_t *status) {
    const uint32_t b = smem_u32(bar);
    if (mbar_try_wait(b, parity)) return true;
    const uint64_t t0 = global_timer();
    while (true) {
        if (mbar_try_wait_sleep(b, parity, 20000u)) return true;
        if (S.abort) return false;
        if (global_timer() - t0 > limit) {
            atomicOr(status, kStatusTimeout);
            S.abort = 1;
            return false;
        }
    }
}

__global__ void __launch_bounds__(kRThreads, 1)
    router_logits_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap,
                         const float *__restrict__ bias, int T, int E, int H, float *__restrict__ lg,
                         uint64_t wait_ns, uint32_t *status) {
    extern __shared__ uint8_t rt_dyn[];
    __shared__ RouteTcShared S;
    const uint32_t pad = (1024u - (smem_u32(rt_dyn) & 1023u)) & 1023u;
    uint8_t *ring = rt_dyn + pad;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * kRM, n0 = blockIdx.y * kRN;
    const int KG = H / kGroup;
    const uint64_t drain_ns = wait_ns > 1000000ull ? wait_ns : 1000000ull;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kRStages; ++s) {
            mbar_init(smem_u32(&S.full[s]), 1);
            mbar_init(smem_u32(&S.empty[s]), 1);
        }
        mbar_init(smem_u32(&S.acc), 1);
        mbar_init(smem_u32(&S.fin), 1);
        S.abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S.tmem)),
                     "r"(kRN)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem;
    if (warp == 0) {
        // ------------------------------------------------------------ tensor copies (one thread)
        if (lane == 0) {
            int kg = 0;
            for (; kg < KG; ++kg) {
                const int s = kg % kRStages;
                if (kg >= kRStages && !rt_wait(S, &S.empty[s], ((kg / kRStages) - 1) & 1u, wait_ns, status)) break;
                const uint32_t fb = smem_u32(&S.full[s]);
                const uint32_t dst = smem_u32(ring + (size_t)s * kRStageBytes);
                mbar_expect_tx(fb, (uint32_t)kRStageBytes);
                tma_load_2d(dst, &xmap, kg * kGroup, m0, fb);
                for (int p = 0; p < kRPlanes; ++p)
                    tma_load_2d(dst + kRABytes + p * kRBBytes, &wmap, kg * kGroup, p * E + n0, fb);
            }
            // copies still in flight land before the CTA may exit
            for (int q = kg > kRStages ? kg - kRStages : 0; q < kg; ++q)
                mbar_wait(smem_u32(&S.full[q % kRStages]), (q / kRStages) & 1u, drain_ns, status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue (one thread)
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kRM, kRN);
            bool ok = true;
            for (int kg = 0; kg < KG && ok; ++kg) {
                const int s = kg % kRStages;
                if (!rt_wait(S, &S.full[s], (kg / kRStages) & 1u, wait_ns, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t As = smem_u32(ring + (size_t)s * kRStageBytes);
#pragma unroll
                for (int p = 0; p < kRPlanes; ++p)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(tmem, sw128_desc(As + 32 * kk), sw128_desc(As + kRABytes + p * kRBBytes + 32 * kk),
                                 idesc, (kg > 0 || p > 0 || kk > 0) ? 1u : 0u);
                umma_commit(smem_u32(&S.empty[s]));
            }
            if (ok) umma_commit(smem_u32(&S.acc));
            // every MMA issued here has completed once `fin` flips (waited for even after an
            // abort, so that TMEM is released only when no MMA still writes it)
            umma_commit(smem_u32(&S.fin));
            mbar_wait(smem_u32(&S.fin), 0, drain_ns, status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue: one token per thread
        const int q = warp & 3;
        const int row = 32 * q + lane, tok = m0 + row;
        if (rt_wait(S, &S.acc, 0, wait_ns, status)) {
            tc_fence_after();
            uint32_t v[4][16];
            const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16);
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld16_nowait(taddr + 16 * c, v[c]);
            tmem_wait_ld();
            if (tok < T) {
                float *dst = lg + (size_t)tok * E + n0;
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int e = n0 + 16 * c + j;
                        if (e < E) dst[16 * c + j] = __uint_as_float(v[c][j]) + (bias ? __ldg(bias + e) : 0.f);
                    }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kRN) : "memory");
}

// top-k + softmax of each token's logits (written by router_logits_kernel), one warp per token
__global__ void topk_from_logits_kernel(const float *lg, int T, int E, int k, int32_t *idx_out, float *w_out) {
    const int lane = threadIdx.x & 31;
    for (int t = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); t < T; t += gridDim.x * (blockDim.x / 32)) {
        int idx;
        float w;
        warp_topk_softmax(lg + (size_t)t * E, true, E, k, lane, idx, w);
        if (lane < k) {
            idx_out[(size_t)t * k + lane] = idx;
            w_out[(size_t)t * k + lane] = w;
        }
    }
}

}  // namespace

// Routing of T tokens through the tensor cores: planes (3 x E x H bf16) and lg (T x E fp32) are
// workspace regions.
moe_status_t launch_route_tc(const uint16_t *x, const float *wr, const float *bias, int T, int H, int E, int k,
                             int32_t *idx_out, float *w_out, uint16_t *planes, float *lg, uint32_t *status,
                             cudaStream_t st) {
    const DeviceInfo *dev = device_info();
    if (!dev) return MOE_ERR_CUDA;
    if (kRSmem + (int)sizeof(RouteTcShared) > dev->max_smem_optin) return MOE_ERR_UNSUPPORTED;
    CUtensorMap xmap, wmap;
    if (!make_tmap_2d_16(&xmap, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, T, H, kRM) ||
        !make_tmap_2d_16(&wmap, planes, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kRPlanes * E, H, kRN))
        return MOE_ERR_CUDA;
    static std::once_flag attr_once[64];
    static bool attr_ok[64] = {};
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64) return MOE_ERR_CUDA;
    std::call_once(attr_once[d], [&] {
        attr_ok[d] = cudaFuncSetAttribute(router_logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRSmem) ==
                     cudaSuccess;
    });
    if (!attr_ok[d]) return MOE_ERR_CUDA;
    const size_t n4 = (size_t)E * H / 4;
    router_split_kernel<<<(unsigned)min((n4 + 255) / 256, (size_t)dev->sms * 8), 256, 0, st>>>(
        reinterpret_cast<const float4 *>(wr), n4, reinterpret_cast<uint2 *>(planes));
    const dim3 grid((unsigned)((T + kRM - 1) / kRM), (unsigned)((E + kRN - 1) / kRN));
    router_logits_kernel<<<grid, kRThreads, kRSmem, st>>>(xmap, wmap, bias, T, E, H, lg, wait_limit_ns(), status);
    topk_from_logits_kernel<<<(unsigned)min((T + 7) / 8, dev->sms * 16), 256, 0, st>>>(lg, T, E, k, idx_out, w_out);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
