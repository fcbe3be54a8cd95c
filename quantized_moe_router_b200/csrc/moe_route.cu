// moe_route.cu -- router logits + top-k + softmax renormalisation for any number of tokens.
//
// One CTA per (up to) 32 tokens computes all E logits l = x W_r^T (+ bias) of its tokens into shared
// memory, then one warp per token runs the top-k + softmax of moe_topk.cuh over them. The logits
// are an fp32 GEMM (fp32 products and sums, as the routing step requires) on the CUDA cores:
// for each chunk of 256 experts the CTA walks H in 32-wide slices; the router rows of the next
// slice stream into shared memory with cp.async (double buffered, no register staging) while x
// of the next slice is widened from bf16 (exact) into the other buffer. Each thread accumulates
// 8 tokens x 4 experts with packed fp32x2 FMAs over pairs of K; its operands are K-contiguous in shared memory,
// so one 16-byte load feeds four K steps (12 loads per 64 FMA pairs per warp). Rows are padded to
// 36 floats and tokens / experts are interleaved across lanes so that every load is free of bank
// conflicts. CTAs start their K walk at different slices (see below).
#include "moe_internal.cuh"
#include "moe_topk.cuh"

namespace moe {
namespace {

constexpr int kRT = 32;    // tokens per CTA
constexpr int kRE = 256;   // experts per chunk
constexpr int kRK = 32;    // K slice
constexpr int kRP = 36;    // padded row (floats)
constexpr int kRThreads = 256;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Thread (warp w, lane = 8 ty + tx) owns tokens ty + 4 i (i < 8) and experts 32 w + tx + 8 j
// (j < 4) of the chunk. Shared memory: logits [kRT][E] | x [2][kRT][kRP] | W [2][kRE][kRP].
__global__ void __launch_bounds__(kRThreads, 1) route_kernel(const uint16_t *__restrict__ x, const float *__restrict__ wr,
                                                             const float *__restrict__ bias, int T, int H, int E, int k,
                                                             int tpc, int32_t *idx_out, float *w_out) {
    extern __shared__ __align__(16) float rsm[];
    float *lg = rsm;                                  // [kRT][E]
    float *xs = rsm + (size_t)kRT * E;                // [2][kRT][kRP]
    float *ws = xs + 2 * kRT * kRP;                   // [2][kRE][kRP]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ty = lane >> 3, tx = lane & 7;
    const int t0 = blockIdx.x * tpc;   // tpc <= kRT tokens per CTA, so that the grid fills the SMs
    const int nt = min(tpc, T - t0);
    const int nslice = H / kRK;
    grid_dep_wait();
    for (int e0 = 0; e0 < E; e0 += kRE) {
        // router rows of slice k0 into buffer b (16-byte pieces; rows past E are not copied and
        // their logits are dropped)
        auto fetch_w = [&](int k0, int b) {
            float *dst = ws + b * kRE * kRP;
#pragma unroll
            for (int r = 0; r < kRE * (kRK / 4) / kRThreads; ++r) {
                const int q = tid + r * kRThreads, e = q >> 3, c = q & 7;
                if (e0 + e < E) cp_async16(smem_u32(dst + e * kRP + 4 * c), wr + (size_t)(e0 + e) * H + k0 + 4 * c);
            }
            cp_async_commit();
        };
        // x of slice k0: thread tid < 128 holds 8 values of token tid / 4
        auto load_x = [&](int k0) -> uint4 {
            const int tk = tid >> 2, kc = (tid & 3) * 8;
            if (tid < 128 && tk < nt) return __ldg(reinterpret_cast<const uint4 *>(x + (size_t)(t0 + tk) * H + k0 + kc));
            return make_uint4(0, 0, 0, 0);
        };
        auto store_x = [&](uint4 v, int b) {
            if (tid < 128) {
                float *dst = xs + b * kRT * kRP + (tid >> 2) * kRP + (tid & 3) * 8;
                *reinterpret_cast<float4 *>(dst) = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                                                               __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u));
                *reinterpret_cast<float4 *>(dst + 4) = make_float4(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xFFFF0000u),
                                                                   __uint_as_float(v.w << 16), __uint_as_float(v.w & 0xFFFF0000u));
            }
        };
        // token i, expert j: the sums over even and over odd K, added at the end; the operand
        // pairs of a packed FMA are then adjacent registers of the 16-byte loads
        float2 acc[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = make_float2(0.f, 0.f);
        // CTA b walks the slices from slice b on (mod the slice count): all CTAs read the same
        // router rows, and in lock step they would queue on the same L2 lines
        const int sl0 = blockIdx.x % nslice;
        auto kof = [&](int sl) { const int q = sl0 + sl; return (q < nslice ? q : q - nslice) * kRK; };
        fetch_w(kof(0), 0);
        store_x(load_x(kof(0)), 0);
        cp_async_wait_all();
        __syncthreads();
        for (int sl = 0; sl < nslice; ++sl) {
            const int cb = sl & 1;
            uint4 xn = make_uint4(0, 0, 0, 0);
            if (sl + 1 < nslice) {
                fetch_w(kof(sl + 1), cb ^ 1);
                xn = load_x(kof(sl + 1));
            }
            const float *xb = xs + cb * kRT * kRP + ty * kRP;
            const float *wb = ws + cb * kRE * kRP + (32 * warp + tx) * kRP;
#pragma unroll 2
            for (int kq = 0; kq < kRK / 4; ++kq) {
                float4 xa[8], wa[4];
#pragma unroll
                for (int i = 0; i < 8; ++i) xa[i] = *reinterpret_cast<const float4 *>(xb + 4 * i * kRP + 4 * kq);
#pragma unroll
                for (int j = 0; j < 4; ++j) wa[j] = *reinterpret_cast<const float4 *>(wb + 8 * j * kRP + 4 * kq);
                // K pair (0, 1) for all 32 accumulators, then pair (2, 3): dependent FMAs are 32 apart
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        acc[i][j] = __ffma2_rn(make_float2(xa[i].x, xa[i].y), make_float2(wa[j].x, wa[j].y), acc[i][j]);
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        acc[i][j] = __ffma2_rn(make_float2(xa[i].z, xa[i].w), make_float2(wa[j].z, wa[j].w), acc[i][j]);
            }
            if (sl + 1 < nslice) store_x(xn, cb ^ 1);
            cp_async_wait_all();
            __syncthreads();
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int tk = ty + 4 * i;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int ee = e0 + 32 * warp + tx + 8 * j;
                const float v = acc[i][j].x + acc[i][j].y;
                if (ee < E) lg[tk * E + ee] = v + (bias ? __ldg(bias + ee) : 0.f);
            }
        }
        __syncthreads();
    }
    for (int i = warp; i < nt; i += kRThreads / 32) {
        int idx;
        float w;
        warp_topk_softmax(lg + (size_t)i * E, false, E, k, lane, idx, w);
        if (lane < k) {
            idx_out[(size_t)(t0 + i) * k + lane] = idx;
            w_out[(size_t)(t0 + i) * k + lane] = w;
        }
    }
}

}  // namespace

moe_status_t launch_route(const uint16_t *x, const float *wr, const float *bias, int T, int H, int E, int k,
                          int32_t *idx_out, float *w_out, cudaStream_t st) {
    const DeviceInfo *dev = device_info();
    if (!dev) return MOE_ERR_CUDA;
    const size_t smem = ((size_t)kRT * E + 2 * (size_t)kRT * kRP + 2 * (size_t)kRE * kRP) * sizeof(float);
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
    // tokens per CTA: as few as fill every SM once, at most kRT
    const int tpc = max(1, min(kRT, (T + dev->sms - 1) / dev->sms));
    const unsigned blocks = (unsigned)((T + tpc - 1) / tpc);
    route_kernel<<<blocks, kRThreads, smem, st>>>(x, wr, bias, T, H, E, k, tpc, idx_out, w_out);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
