// moe_decode.cu -- the decode megakernel: one persistent launch per layer computes routing,
// gate/up, SiLU-GLU, down and the weighted combine of the MoE expert block for T <= 32 tokens.
//
// This is the "MoE megakernel" of the page "Raon-1-mini ... RTX 5070 Ti" (table row: one
// persistent kernel for each layer's expert block) with the "pipelined megakernel" row's
// overlap (the next expert's tiles are in flight while the current one computes), designed
// for sm_100a:
//   * one CTA per SM, 8 consumer warps + 1 producer warp;
//   * phase R: each CTA computes the fp32 router logits of E/nCTA experts, zeroes its share of
//     the fp32 accumulators and the per-group sums of x, then a bounded grid barrier;
//   * every CTA reads all logits from L2 and runs the same warp top-k + softmax, so all CTAs
//     agree on the selected experts without a second exchange;
//   * phase X: the selected experts' packed tiles are split into gate/up jobs (8 intermediate
//     rows x all of H) and down jobs (16 output rows x all of I), statically balanced over CTAs
//     by bytes; the producer streams each job's tiles with 1-D bulk copies (no multicast) into
//     a 6-stage ring guarded by mbarriers, and each consumer warp multiplies one tile per stage
//     with mma.sync on bf16 operands made from the 4-bit codes by one LOP3 per register (exact
//     integers 128+q), applying the group's scale and zero to the fp32 partial sums;
//   * gate/up jobs finish with SiLU-GLU and write h (split into bf16 hi + lo, exact to 2^-17)
//     and its group sums; a second bounded grid barrier makes h visible; down jobs add
//     w_i * y into an fp32 accumulator with red.add; the last CTA to finish converts it to
//     bf16. The down tiles are already streaming while the barrier is pending.
#include <cstdio>
#include "moe_internal.cuh"
#include "moe_topk.cuh"

namespace moe {
namespace {

constexpr int kCW = 8;                      // consumer warps
constexpr int kThreads = (kCW + 1) * 32;    // + one producer warp
constexpr int kStageTiles = kCW;            // one tile per consumer warp per stage
constexpr int kStageBytes = kStageTiles * tile_bytes(8);
constexpr int kStages = 6;
constexpr int kMaxP = 256;                  // decode limit on T*k

struct DecodeArgs {
    const uint16_t *x;
    const float *wr;
    const float *bias;
    const uint8_t *packed;
    int T, H, I, E, k;
    uint16_t *out;
    int32_t *idx_out;
    float *w_out;
    Control *ctl;
    float *logits;
    uint16_t *h_hi, *h_lo;
    float *hsum, *out_acc;
    uint64_t wait_ns;
};

struct __align__(16) DecodeSmem {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    int U, nGUc, nDc, d_start, d_stride, abort, is_last, uniform_bits;
    uint32_t selmask[kMaxE / 32];
    int wordpre[kMaxE / 32];
    int ue[kMaxP];
    int ubits[kMaxP];
    unsigned long long uoff[kMaxP];
    int cnt[kMaxP];
    int pfirst[kMaxP + 1];
    int cursor[kMaxP];
    int ptok[kMaxP];
    int ppair[kMaxP];
    float pw[kMaxP];
    int sel_idx[kMaxP];
    float sel_w[kMaxP];
};

__host__ __device__ inline int nt_max(int T) { return (T + 7) / 8; }

size_t decode_smem_bytes(int T, int H) {
    size_t o = align_up(sizeof(DecodeSmem), 128);
    o += (size_t)kStages * kStageBytes;
    o += align_up((size_t)T * (H / kGroup) * 4, 16);
    o += (size_t)2 * kCW * nt_max(T) * 32 * 4 * 4;
    return o;
}

__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ int slot_of(const DecodeSmem &S, int e) {
    const int w = e >> 5;
    return S.wordpre[w] + __popc(S.selmask[w] & ((1u << (e & 31)) - 1u));
}

struct Job {
    const uint8_t *src;
    int ntiles;  // tiles in this job
    int tb;      // bytes per tile
    int bits;
    int u;       // unique-expert slot
    int rb;      // row block
    bool gu;
};

__device__ __forceinline__ Job job_at(const DecodeSmem &S, const DecodeArgs &a, int n, int c, int nC) {
    Job j;
    const int G = a.H / kGroup, GI = a.I / kGroup;
    if (n < S.nGUc) {
        const int gj = c + n * nC;
        const int rbg = a.I / 8;
        j.u = gj / rbg;
        j.rb = gj % rbg;
        j.gu = true;
        j.ntiles = G;
    } else {
        const int d = S.d_start + (n - S.nGUc) * S.d_stride;
        const int rbd = a.H / 16;
        j.u = d / rbd;
        j.rb = d % rbd;
        j.gu = false;
        j.ntiles = GI;
    }
    j.bits = S.ubits[j.u];
    j.tb = tile_bytes(j.bits);
    const uint8_t *base = a.packed + S.uoff[j.u];
    if (j.gu)
        j.src = base + (size_t)j.rb * G * j.tb;
    else
        j.src = base + gu_tiles(a.H, a.I) * j.tb + (size_t)j.rb * GI * j.tb;
    return j;
}

// One tile (one quantisation group) of a job for every n-tile of the job's tokens.
template <int BITS>
__device__ __forceinline__ void consume_tile(const DecodeArgs &a, const DecodeSmem &S,
                                             const uint8_t *tile, const Job &jb, int kg,
                                             const float *Xs, int lane, float (&acc)[4][4]) {
    const int g = lane >> 2, t = lane & 3;
    const uint4 lo = *reinterpret_cast<const uint4 *>(tile + 16 * lane);
    uint4 hi8 = make_uint4(0, 0, 0, 0);
    uint2 hi6 = make_uint2(0, 0);
    if (BITS == 8) hi8 = *reinterpret_cast<const uint4 *>(tile + kLoBytes + 16 * lane);
    if (BITS == 6) hi6 = *reinterpret_cast<const uint2 *>(tile + kLoBytes + 8 * lane);
    const uint2 sz = *reinterpret_cast<const uint2 *>(tile + kLoBytes + hi_bytes(BITS) + 8 * g);
    const float sA = half_lo(sz.x), zA = half_hi(sz.x), sB = half_lo(sz.y), zB = half_hi(sz.y);
    const int pf = S.pfirst[jb.u];
    const int nu = S.pfirst[jb.u + 1] - pf;
    const int G = a.H / kGroup, GI = a.I / kGroup;
    const int ntn = (nu + 7) >> 3;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        if (nt >= ntn) break;
        const int q = nt * 8 + g, q0 = nt * 8 + 2 * t, q1 = q0 + 1;
        uint32_t b[8] = {0, 0, 0, 0, 0, 0, 0, 0}, b2[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        float X0 = 0.f, X1 = 0.f;
        if (jb.gu) {
            if (q < nu) {
                const uint4 *xp = reinterpret_cast<const uint4 *>(a.x + (size_t)S.ptok[pf + q] * a.H +
                                                                  kg * kGroup + 16 * t);
                const uint4 xa = __ldg(xp), xb = __ldg(xp + 1);
                b[0] = xa.x; b[1] = xa.y; b[2] = xa.z; b[3] = xa.w;
                b[4] = xb.x; b[5] = xb.y; b[6] = xb.z; b[7] = xb.w;
            }
            if (q0 < nu) X0 = Xs[S.ptok[pf + q0] * G + kg];
            if (q1 < nu) X1 = Xs[S.ptok[pf + q1] * G + kg];
            tile_group_mma<BITS>(lo, hi8, hi6, b, nullptr, sA, zA, sB, zB, X0, X1, acc[nt]);
        } else {
            if (q < nu) {
                const size_t off = (size_t)S.ppair[pf + q] * a.I + kg * kGroup + 16 * t;
                const uint4 *hp = reinterpret_cast<const uint4 *>(a.h_hi + off);
                const uint4 *lp = reinterpret_cast<const uint4 *>(a.h_lo + off);
                const uint4 ha = __ldcg(hp), hb = __ldcg(hp + 1), la = __ldcg(lp), lb = __ldcg(lp + 1);
                b[0] = ha.x; b[1] = ha.y; b[2] = ha.z; b[3] = ha.w;
                b[4] = hb.x; b[5] = hb.y; b[6] = hb.z; b[7] = hb.w;
                b2[0] = la.x; b2[1] = la.y; b2[2] = la.z; b2[3] = la.w;
                b2[4] = lb.x; b2[5] = lb.y; b2[6] = lb.z; b2[7] = lb.w;
            }
            if (q0 < nu) X0 = __ldcg(a.hsum + (size_t)S.ppair[pf + q0] * GI + kg);
            if (q1 < nu) X1 = __ldcg(a.hsum + (size_t)S.ppair[pf + q1] * GI + kg);
            tile_group_mma<BITS>(lo, hi8, hi6, b, b2, sA, zA, sB, zB, X0, X1, acc[nt]);
        }
    }
}

__device__ void job_epilogue(const DecodeArgs &a, const DecodeSmem &S, const Job &jb, float *red,
                             int NTM, int warp, int lane, float (&acc)[4][4]) {
    const int pf = S.pfirst[jb.u];
    const int nu = S.pfirst[jb.u + 1] - pf;
    const int ntn = (nu + 7) >> 3;
    for (int nt = 0; nt < ntn; ++nt)
        *reinterpret_cast<float4 *>(red + ((warp * NTM + nt) * 32 + lane) * 4) =
            make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
    consumer_sync();
    if (warp != 0) return;
    const int g = lane >> 2, t = lane & 3;
    const int GI = a.I / kGroup;
    for (int nt = 0; nt < ntn; ++nt) {
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        for (int w = 0; w < kCW; ++w) {
            const float4 p = *reinterpret_cast<const float4 *>(red + ((w * NTM + nt) * 32 + lane) * 4);
            v[0] += p.x; v[1] += p.y; v[2] += p.z; v[3] += p.w;
        }
        for (int col = 0; col < 2; ++col) {
            const int q = nt * 8 + 2 * t + col;
            const bool valid = q < nu;
            if (jb.gu) {
                const float gate = v[col], up = v[2 + col];
                const float h = gate / (1.f + expf(-gate)) * up;
                const __nv_bfloat16 hi = __float2bfloat16_rn(h);
                const __nv_bfloat16 lo = __float2bfloat16_rn(h - __bfloat162float(hi));
                float part = 0.f;
                int pair = 0;
                if (valid) {
                    pair = S.ppair[pf + q];
                    const size_t o = (size_t)pair * a.I + jb.rb * 8 + g;
                    a.h_hi[o] = __bfloat16_as_ushort(hi);
                    a.h_lo[o] = __bfloat16_as_ushort(lo);
                    part = __bfloat162float(hi) + __bfloat162float(lo);
                }
                part += __shfl_xor_sync(0xffffffffu, part, 4);
                part += __shfl_xor_sync(0xffffffffu, part, 8);
                part += __shfl_xor_sync(0xffffffffu, part, 16);
                if (g == 0 && valid) red_add_f32(a.hsum + (size_t)pair * GI + (jb.rb >> 3), part);
            } else if (valid) {
                const int tok = S.ptok[pf + q];
                const float wgt = S.pw[pf + q];
                const int row = jb.rb * 16 + g;
                red_add_f32(a.out_acc + (size_t)tok * a.H + row, wgt * v[col]);
                red_add_f32(a.out_acc + (size_t)tok * a.H + row + 8, wgt * v[2 + col]);
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t dyn[];
    DecodeSmem &S = *reinterpret_cast<DecodeSmem *>(dyn);
    uint8_t *stages = dyn + align_up(sizeof(DecodeSmem), 128);
    float *Xs = reinterpret_cast<float *>(stages + (size_t)kStages * kStageBytes);
    const int T = a.T, H = a.H, I = a.I, E = a.E, K = a.k, P = T * K;
    const int G = H / kGroup, GI = I / kGroup;
    float *redbuf = Xs + align_up((size_t)T * G, 4);
    const int NTM = nt_max(T);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nC = gridDim.x, c = blockIdx.x;
    uint32_t *status = &a.ctl->status;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&S.full[s]), 1);
            mbar_init(smem_u32(&S.empty[s]), kCW);
        }
        fence_barrier_init();
        S.abort = 0;
        S.is_last = 0;
    }
    for (int i = threadIdx.x; i < kMaxE / 32; i += kThreads) S.selmask[i] = 0;
    __syncthreads();
    // Everything below reads data that the previous launch in the stream may produce.
    grid_dep_wait();

    // ---------------------------------------------------------------- phase R
    const int gtid = c * kThreads + threadIdx.x, gthreads = nC * kThreads;
    for (int i = gtid; i < T * H; i += gthreads) a.out_acc[i] = 0.f;
    for (int i = gtid; i < P * GI; i += gthreads) a.hsum[i] = 0.f;
    const int ne = (E > c) ? (E - c + nC - 1) / nC : 0;
    for (int q = warp; q < ne * T; q += kCW + 1) {
        const int e = c + (q / T) * nC, t = q % T;
        const float *wrow = a.wr + (size_t)e * H;
        const uint16_t *xrow = a.x + (size_t)t * H;
        float acc = 0.f;
        for (int h = lane * 8; h < H; h += 256) {
            const float4 w0 = __ldg(reinterpret_cast<const float4 *>(wrow + h));
            const float4 w1 = __ldg(reinterpret_cast<const float4 *>(wrow + h + 4));
            const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(xrow + h));
            acc += w0.x * __uint_as_float(xv.x << 16) + w0.y * __uint_as_float(xv.x & 0xFFFF0000u);
            acc += w0.z * __uint_as_float(xv.y << 16) + w0.w * __uint_as_float(xv.y & 0xFFFF0000u);
            acc += w1.x * __uint_as_float(xv.z << 16) + w1.y * __uint_as_float(xv.z & 0xFFFF0000u);
            acc += w1.z * __uint_as_float(xv.w << 16) + w1.w * __uint_as_float(xv.w & 0xFFFF0000u);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) a.logits[(size_t)t * E + e] = acc + (a.bias ? a.bias[e] : 0.f);
    }
    for (int i = threadIdx.x; i < T * G; i += kThreads) {
        const int t = i / G, gq = i % G;
        const uint16_t *xp = a.x + (size_t)t * H + gq * kGroup;
        float s = 0.f;
        for (int j = 0; j < kGroup; ++j) s += bf16_bits_to_float(xp[j]);
        Xs[i] = s;
    }
    __syncthreads();
    if (threadIdx.x == 0 && !grid_barrier(&a.ctl->bar, nC, c == 0, a.wait_ns, status)) S.abort = 1;
    __syncthreads();
    grid_dep_launch();

    // ---------------------------------------------------------------- routing
    if (!S.abort) {
        for (int t = warp; t < T; t += kCW + 1) {
            int idx;
            float w;
            warp_topk_softmax(a.logits + (size_t)t * E, true, E, K, lane, idx, w);
            if (lane < K) {
                S.sel_idx[t * K + lane] = idx;
                S.sel_w[t * K + lane] = w;
                if (c == 0 && a.idx_out) a.idx_out[t * K + lane] = idx;
                if (c == 0 && a.w_out) a.w_out[t * K + lane] = w;
            }
        }
    }
    __syncthreads();
    const bool aborted = S.abort != 0;
    if (!aborted)
        for (int p = threadIdx.x; p < P; p += kThreads)
            atomicOr(&S.selmask[S.sel_idx[p] >> 5], 1u << (S.sel_idx[p] & 31));
    __syncthreads();
    if (warp == 0) {
        const int words = (E + 31) / 32;
        const int n = (lane < words) ? __popc(S.selmask[lane]) : 0;
        int incl = n;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
        }
        S.wordpre[lane] = incl - n;
        if (lane == 31) S.U = incl;
    }
    __syncthreads();
    const PackedExpert *pe = reinterpret_cast<const PackedExpert *>(a.packed + sizeof(PackedHeader));
    for (int e = threadIdx.x; e < E; e += kThreads) {
        if ((S.selmask[e >> 5] >> (e & 31)) & 1u) {
            const int s = slot_of(S, e);
            S.ue[s] = e;
            S.ubits[s] = pe[e].bits;
            S.uoff[s] = pe[e].offset;
            S.cnt[s] = 0;
        }
    }
    __syncthreads();
    for (int p = threadIdx.x; p < (aborted ? 0 : P); p += kThreads) atomicAdd(&S.cnt[slot_of(S, S.sel_idx[p])], 1);
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < S.U; base += 32) {
            const int s = base + lane;
            const int n = (s < S.U) ? S.cnt[s] : 0;
            int incl = n;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o;
            }
            if (s < S.U) {
                S.pfirst[s] = carry + incl - n;
                S.cursor[s] = carry + incl - n;
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) S.pfirst[S.U] = carry;
        __syncwarp();
        // stable fill: pairs in ascending pair id (token-major) order
        for (int base = 0; base < (aborted ? 0 : P); base += 32) {
            const int p = base + lane;
            const int s = (p < P) ? slot_of(S, S.sel_idx[p]) : -1 - lane;
            const uint32_t peers = __match_any_sync(0xffffffffu, s);
            const int rank = __popc(peers & ((1u << lane) - 1u));
            if (p < P) {
                const int pos = S.cursor[s] + rank;
                S.ppair[pos] = p;
                S.ptok[pos] = p / K;
                S.pw[pos] = S.sel_w[p];
            }
            __syncwarp();
            if (p < P && rank == 0) S.cursor[s] += __popc(peers);
            __syncwarp();
        }
        // job plan
        if (lane == 0) {
            int U = aborted ? 0 : S.U;
            int ub = U > 0 ? S.ubits[0] : 4;
            for (int s = 1; s < U; ++s)
                if (S.ubits[s] != ub) ub = 0;
            S.uniform_bits = ub;
            const long long nGU = (long long)U * (I / 8), nD = (long long)U * (H / 16);
            S.nGUc = (nGU > c) ? (int)((nGU - c + nC - 1) / nC) : 0;
            const long long q = nGU / nC, r = nGU % nC;
            const long long W = nGU * G + nD * GI;  // in tiles (uniform width)
            bool balanced = ub != 0 && (long long)nC * (q + 1) * G <= W;
            if (balanced) {
                const long long d1 = (W - (long long)nC * (q + 1) * G) / ((long long)nC * GI);
                const long long d0 = (W - (long long)nC * q * G) / ((long long)nC * GI);
                const long long L = nD - r * d1 - (nC - r) * d0;
                const long long e0 = L < (nC - r) ? L : (nC - r);
                const long long L1 = L - e0;
                if (L < 0 || L1 > r) balanced = false;
                if (balanced) {
                    long long cnt, start;
                    if (c < r) {
                        cnt = d1 + (c < L1 ? 1 : 0);
                        start = (long long)c * d1 + (c < L1 ? c : L1);
                    } else {
                        cnt = d0 + ((c - r) < e0 ? 1 : 0);
                        start = r * d1 + L1 + (c - r) * d0 + ((c - r) < e0 ? (c - r) : e0);
                    }
                    S.d_start = (int)start;
                    S.d_stride = 1;
                    S.nDc = (int)cnt;
                }
            }
            if (!balanced) {
                const int st = (int)(((c - r) % nC + nC) % nC);
                S.d_start = st;
                S.d_stride = nC;
                S.nDc = (nD > st) ? (int)((nD - st + nC - 1) / nC) : 0;
            }
        }
    }
    __syncthreads();

    const int njobs = S.nGUc + S.nDc;
    if (warp == kCW) {
        // ------------------------------------------------------------ producer
        if (lane != 0) return;
        uint32_t cc = 0;
        for (int n = 0; n < njobs; ++n) {
            const Job jb = job_at(S, a, n, c, nC);
            for (int c0 = 0; c0 < jb.ntiles; c0 += kStageTiles) {
                const int s = cc % kStages;
                const uint32_t use = cc / kStages;
                if (use > 0 && !mbar_wait(smem_u32(&S.empty[s]), (use - 1) & 1u, a.wait_ns, status)) return;
                const int nt = min(kStageTiles, jb.ntiles - c0);
                const uint32_t bytes = (uint32_t)(nt * jb.tb);
                const uint32_t fb = smem_u32(&S.full[s]);
                mbar_expect_tx(fb, bytes);
                bulk_g2s(smem_u32(stages + (size_t)s * kStageBytes), jb.src + (size_t)c0 * jb.tb, bytes, fb);
                ++cc;
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    uint32_t cc = 0;
    bool skip = aborted;
    for (int n = 0; n < njobs; ++n) {
        if (n == S.nGUc) {
            // all h written by every CTA before any down job reads it
            __threadfence();
            consumer_sync();
            if (threadIdx.x == 0 && !grid_barrier(&a.ctl->bar, nC, c == 0, a.wait_ns, status)) S.abort = 1;
            consumer_sync();
            skip = skip || (S.abort != 0);
        }
        const Job jb = job_at(S, a, n, c, nC);
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
        for (int c0 = 0; c0 < jb.ntiles; c0 += kStageTiles) {
            const int s = cc % kStages;
            const uint32_t use = cc / kStages;
            if (!mbar_wait(smem_u32(&S.full[s]), use & 1u, a.wait_ns, status)) return;
            const int kg = c0 + warp;
            if (!skip && kg < jb.ntiles) {
                const uint8_t *tile = stages + (size_t)s * kStageBytes + (size_t)warp * jb.tb;
                if (jb.bits == 4)
                    consume_tile<4>(a, S, tile, jb, kg, Xs, lane, acc);
                else if (jb.bits == 6)
                    consume_tile<6>(a, S, tile, jb, kg, Xs, lane, acc);
                else
                    consume_tile<8>(a, S, tile, jb, kg, Xs, lane, acc);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&S.empty[s]));
            ++cc;
        }
        if (!skip) job_epilogue(a, S, jb, redbuf + (size_t)(n & 1) * kCW * NTM * 32 * 4, NTM, warp, lane, acc);
    }
    if (S.nGUc == njobs) {
        // a CTA without down jobs still takes part in the second grid barrier
        __threadfence();
        consumer_sync();
        if (threadIdx.x == 0 && !grid_barrier(&a.ctl->bar, nC, c == 0, a.wait_ns, status)) S.abort = 1;
        consumer_sync();
    }
    // ---------------------------------------------------------------- completion
    __threadfence();
    consumer_sync();
    if (threadIdx.x == 0) {
        const uint32_t old = atom_add_acq_rel(&a.ctl->done, 1u);
        S.is_last = (old == (uint32_t)nC - 1u);
    }
    consumer_sync();
    if (S.is_last) {
        __threadfence();
        for (int i = threadIdx.x; i < T * H; i += kCW * 32)
            a.out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(__ldcg(a.out_acc + i)));
        if (threadIdx.x == 0) a.ctl->done = 0;
    }
}

}  // namespace

moe_status_t launch_decode(const uint16_t *x, const float *wr, const float *bias, const void *packed,
                           int T, int H, int I, int E, int k, uint16_t *out, int32_t *idx_out,
                           float *w_out, void *ws, cudaStream_t st) {
    if (T * k > kMaxP) return MOE_ERR_UNSUPPORTED;
    const DeviceInfo *dev = device_info();
    const DecodeWs L = decode_ws_layout(T, H, I, E, k);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    DecodeArgs a;
    a.x = x; a.wr = wr; a.bias = bias; a.packed = static_cast<const uint8_t *>(packed);
    a.T = T; a.H = H; a.I = I; a.E = E; a.k = k;
    a.out = out; a.idx_out = idx_out; a.w_out = w_out;
    a.ctl = reinterpret_cast<Control *>(w8);
    a.logits = reinterpret_cast<float *>(w8 + L.logits);
    a.h_hi = reinterpret_cast<uint16_t *>(w8 + L.h_hi);
    a.h_lo = reinterpret_cast<uint16_t *>(w8 + L.h_lo);
    a.hsum = reinterpret_cast<float *>(w8 + L.hsum);
    a.out_acc = reinterpret_cast<float *>(w8 + L.out_acc);
    a.wait_ns = wait_limit_ns();
    const size_t smem = decode_smem_bytes(T, H);
    if ((int)smem > dev->max_smem_optin) return MOE_ERR_UNSUPPORTED;
    static bool attr_set[16] = {false};
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) return MOE_ERR_CUDA;
    if (d < 16 && !attr_set[d]) {
        if (cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dev->max_smem_optin) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_set[d] = true;
    }
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel, kThreads, smem) != cudaSuccess ||
        per_sm < 1)
        return MOE_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(dev->sms);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, decode_kernel, a) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

}  // namespace moe
