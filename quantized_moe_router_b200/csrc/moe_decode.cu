// moe_decode.cu -- the decode megakernel: one persistent launch per layer computes routing,
// gate/up, SiLU-GLU, down and the weighted combine of the MoE expert block for T <= 32 tokens.
//
// This is the "MoE megakernel" of the page "Raon-1-mini ... RTX 5070 Ti" (table row: one
// persistent kernel for each layer's expert block) with the "pipelined megakernel" row's
// overlap (the next expert's tiles are in flight while the current one computes), designed
// for sm_100a:
//   * one CTA per SM, 8 consumer warps + 1 producer warp;
//   * prologue, before the programmatic-dependent-launch wait so that it overlaps the previous
//     layer: barrier set-up, this CTA's router rows copied to shared memory, the packed layer's
//     expert table read (both are weights, never produced by the previous launch);
//   * phase R: x is copied to shared memory, each CTA computes the fp32 router logits of its
//     E/nCTA experts, zeroes its share of the fp32 accumulators and the per-group sums of x,
//     then a bounded grid barrier;
//   * every CTA reads all logits from L2 and runs the same CTA-wide top-k + softmax (each warp
//     selects within a slice of the experts, then every candidate's rank is counted in
//     parallel), so all CTAs agree on the selected experts without a second exchange;
//   * phase X: the selected experts' packed tiles form two job sequences, gate/up jobs
//     (8 intermediate rows x all of H) and down jobs (16 output rows x all of I). Each CTA gets
//     a contiguous range of each, cut so that every CTA streams the same number of bytes, so
//     its data is a few long contiguous regions. The producer streams them in 24 KB bulk
//     copies (on B200 one SM completes roughly one bulk copy per ~250 ns whatever its size,
//     so copies must be large to reach HBM bandwidth) into a 4-stage ring. Tiles go
//     round-robin to the 8 consumer warps, which multiply them with mma.sync on bf16
//     operands made from the codes by one LOP3 per register (exact integers 128+q) and apply
//     the group's scale and zero to fp32 partial sums;
//   * gate/up partial sums are combined without CTA barriers: each warp flushes its partial of
//     a job into a shared-memory slot and the last of the 8 warps to flush applies SiLU-GLU and
//     writes h (bf16 hi + lo, exact to 2^-17) and its group sums;
//   * a second bounded grid barrier makes h visible; each CTA loads h into shared memory; down
//     jobs add w_i * y into an fp32 accumulator with red.add; the last CTA to finish converts
//     it to bf16. The down tiles stream in while the barrier is pending.
// The kernel is instantiated for 1, 2 and 4 MMA n-tiles (up to 8, 16 and 32 tokens per expert).
#include "moe_internal.cuh"
#include "moe_topk.cuh"

namespace moe {
namespace {

constexpr int kCW = 8;                      // consumer warps
constexpr int kWarps = kCW + 2;             // + one producer warp + one gate/up epilogue warp
constexpr int kThreads = kWarps * 32;
constexpr int kStageBytes = 24576;          // bytes per bulk copy / pipeline stage
constexpr int kStages = 4;
constexpr int kActBytes = 49152;            // smem for x (routing + gate/up), then h (down)
constexpr int kRedBytes = 32768;            // gate/up partial-sum slots (top-k scratch before)
constexpr int kHStageBytes = 16384;         // finished h of this CTA's gate/up jobs, written out in one burst
constexpr int kMaxP = 256;                  // decode limit on T*k
constexpr int kSlices = 8;                  // expert slices of the first top-k stage

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
    uint64_t wbar, xbar;
    int U, abort, is_last, nGUc;
    int g0, g1, d0, d1;                 // this CTA's gate/up and down job ranges
    int slot_cnt[8];
    int slot_seq[8];
    uint32_t eoff[kMaxE];               // packed offset / 256 of every expert
    uint8_t ebits[kMaxE];               // code width of every expert
    uint32_t selmask[kMaxE / 32];
    int wordpre[kMaxE / 32];
    int ubits[kMaxP];
    uint32_t uoff[kMaxP];
    int cnt[kMaxP];
    int pfirst[kMaxP + 1];
    int cursor[kMaxP];
    uint32_t cgu[kMaxP + 1];            // 64-byte units of all gate/up jobs of expert slots < u
    uint32_t cd[kMaxP + 1];             // 64-byte units of all down jobs of expert slots < u
    int ptok[kMaxP];
    int ppair[kMaxP];
    float pw[kMaxP];
    int sel_idx[kMaxP];
    uint32_t sel_key[kMaxP];
    float sel_w[kMaxP];
};

size_t decode_smem_bytes(int T, int H) {
    size_t o = align_up(sizeof(DecodeSmem), 128);
    o += (size_t)kStages * kStageBytes + kActBytes + kRedBytes + kHStageBytes;
    o += align_up((size_t)T * (H / kGroup) * 4, 16);
    return o;
}

__host__ __device__ inline bool x_in_smem(int T, int H) { return (size_t)T * H * 2 <= (size_t)kActBytes; }
__host__ __device__ inline size_t h_smem_bytes(int P, int I) {
    return (size_t)2 * P * I * 2 + align_up((size_t)P * (I / kGroup) * 4, 16);
}

__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
// consumers + the epilogue warp: every gate/up job of the CTA is finalised
__device__ __forceinline__ void gu_done_sync() { asm volatile("bar.sync 2, 288;" ::: "memory"); }
// CTA-scope acquire / release on shared-memory words (hand-off of partial sums between warps)
__device__ __forceinline__ int ld_acquire_cta(const int *p) {
    int v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_cta(int *p, int v) {
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ int atom_add_acq_rel_cta(int *p, int v) {
    int old;
    asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(smem_u32(p)), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ int slot_of(const DecodeSmem &S, int e) {
    const int w = e >> 5;
    return S.wordpre[w] + __popc(S.selmask[w] & ((1u << (e & 31)) - 1u));
}

// ------------------------------------------------------------------------------ job layout
// A run of consecutive jobs of one expert and one phase: contiguous in the packed layer.
struct Region {
    const uint8_t *src;
    int tiles, tb, bits, u, rb0, job0, tpj;   // job0: CTA-local index of the first job
};

__device__ __forceinline__ Region region_at(const DecodeSmem &S, const DecodeArgs &a, bool gu, int j) {
    Region r;
    const int G = a.H / kGroup, GI = a.I / kGroup;
    const int per = gu ? a.I / 8 : a.H / 16;    // jobs per expert
    const int end = gu ? S.g1 : S.d1;
    r.u = j / per;
    r.rb0 = j % per;
    const int jend = min(end, (r.u + 1) * per);
    r.tpj = gu ? G : GI;
    r.tiles = (jend - j) * r.tpj;
    r.bits = S.ubits[r.u];
    r.tb = tile_bytes(r.bits);
    r.job0 = gu ? (j - S.g0) : (S.nGUc + j - S.d0);
    const uint8_t *base = a.packed + (size_t)S.uoff[r.u] * 256;
    r.src = gu ? base + (size_t)r.rb0 * G * r.tb : base + gu_tiles(a.H, a.I) * r.tb + (size_t)r.rb0 * GI * r.tb;
    return r;
}
__device__ __forceinline__ int region_chunks(const Region &r) {
    const int cap = kStageBytes / r.tb;
    return (r.tiles + cap - 1) / cap;
}
// tiles [c0, c0 + m) of chunk i of a region (balanced split)
__device__ __forceinline__ void chunk_range(const Region &r, int n, int i, int &c0, int &m) {
    const int base = r.tiles / n, rem = r.tiles % n;
    m = base + (i < rem ? 1 : 0);
    c0 = i * base + (i < rem ? i : rem);
}

// First job (of the gate/up or down sequence) whose first 64-byte unit is at or after `pos`;
// cum[u] = units of the jobs of expert slots < u, `per` jobs per expert.
__device__ __forceinline__ int job_at_unit(const uint32_t *cum, int U, int per, uint32_t pos) {
    if (pos == 0) return 0;
    if (pos >= cum[U]) return U * per;
    int lo = 0, hi = U;                 // largest u with cum[u] <= pos
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cum[mid] <= pos) lo = mid; else hi = mid;
    }
    const uint32_t jb = (cum[lo + 1] - cum[lo]) / per;   // units per job of expert lo
    return lo * per + (int)((pos - cum[lo] + jb - 1) / jb);
}
__device__ __forceinline__ uint32_t job_start_unit(const uint32_t *cum, int U, int per, int j) {
    if (j >= U * per) return cum[U];
    const int u = j / per;
    return cum[u] + (cum[u + 1] - cum[u]) / per * (uint32_t)(j % per);
}

// ------------------------------------------------------------------------------ tile math
// Operand sources of the current job for this lane: per n-tile, the row of x (gate/up) or of
// h hi / lo (down) that the lane's B column reads, and the rows of group sums of its two
// accumulator columns (null where the column has no token).
template <int NT>
struct JobCtx {
    const uint16_t *b[NT];
    const uint16_t *b2[NT];
    const float *xs0[NT];
    const float *xs1[NT];
};

template <int BITS, int NT, bool GU>
__device__ __forceinline__ void consume_tile(const uint8_t *tile, int kg, const JobCtx<NT> &jc, int lane,
                                             float (&acc)[NT][4], float keep = 1.f) {
    const int g = lane >> 2, t = lane & 3;
    const uint4 lo = *reinterpret_cast<const uint4 *>(tile + 16 * lane);
    uint4 hi8 = make_uint4(0, 0, 0, 0);
    uint2 hi6 = make_uint2(0, 0);
    if (BITS == 8) hi8 = *reinterpret_cast<const uint4 *>(tile + kLoBytes + 16 * lane);
    if (BITS == 6) hi6 = *reinterpret_cast<const uint2 *>(tile + kLoBytes + 8 * lane);
    const uint2 sz = *reinterpret_cast<const uint2 *>(tile + kLoBytes + hi_bytes(BITS) + 8 * g);
    // keep = 0 turns the tile into a no-op (scales zeroed), so that pairs of tiles run without a
    // branch and their MMA chains interleave
    const float sA = keep * half_lo(sz.x), zA = half_hi(sz.x), sB = keep * half_lo(sz.y), zB = half_hi(sz.y);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        uint32_t b[8] = {0, 0, 0, 0, 0, 0, 0, 0}, b2[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (jc.b[nt]) {
            const uint16_t *p = jc.b[nt] + kg * kGroup + 16 * t;
            const uint4 v0 = *reinterpret_cast<const uint4 *>(p), v1 = *reinterpret_cast<const uint4 *>(p + 8);
            b[0] = v0.x; b[1] = v0.y; b[2] = v0.z; b[3] = v0.w;
            b[4] = v1.x; b[5] = v1.y; b[6] = v1.z; b[7] = v1.w;
            if (!GU) {
                const uint16_t *p2 = jc.b2[nt] + kg * kGroup + 16 * t;
                const uint4 w0 = *reinterpret_cast<const uint4 *>(p2), w1 = *reinterpret_cast<const uint4 *>(p2 + 8);
                b2[0] = w0.x; b2[1] = w0.y; b2[2] = w0.z; b2[3] = w0.w;
                b2[4] = w1.x; b2[5] = w1.y; b2[6] = w1.z; b2[7] = w1.w;
            }
        }
        const float X0 = jc.xs0[nt] ? jc.xs0[nt][kg] : 0.f;
        const float X1 = jc.xs1[nt] ? jc.xs1[nt][kg] : 0.f;
        tile_group_mma<BITS>(lo, hi8, hi6, b, GU ? nullptr : b2, sA, zA, sB, zB, X0, X1, acc[nt]);
    }
}

// SiLU-GLU of a finished gate/up job from the 8 warps' partials in slot `red`. With `stage`
// set, h (bf16 hi + lo of the lane's two columns) goes to shared memory and is written out
// after the gate/up phase (a warp with global writes in flight makes every later CTA-scope
// fence wait for them); otherwise h and its group sums go straight to global memory.
template <int NT>
__device__ void gu_finalize(const DecodeArgs &a, const DecodeSmem &S, int u, int rb, const float *red, int lane,
                            uint2 *stage) {
    const int pf = S.pfirst[u];
    const int nu = S.pfirst[u + 1] - pf;
    const int g = lane >> 2, t = lane & 3;
    const int GI = a.I / kGroup;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int w = 0; w < kCW; ++w) {
            const float4 p = *reinterpret_cast<const float4 *>(red + ((w * NT + nt) * 32 + lane) * 4);
            v[0] += p.x; v[1] += p.y; v[2] += p.z; v[3] += p.w;
        }
        uint32_t his = 0, los = 0;
#pragma unroll
        for (int col = 0; col < 2; ++col) {
            const int q = nt * 8 + 2 * t + col;
            const bool valid = q < nu;
            const float gate = v[col], up = v[2 + col];
            const float h = __fdividef(gate, 1.f + __expf(-gate)) * up;
            const __nv_bfloat16 hi = __float2bfloat16_rn(h);
            const __nv_bfloat16 lo = __float2bfloat16_rn(h - __bfloat162float(hi));
            his |= (uint32_t)__bfloat16_as_ushort(hi) << (16 * col);
            los |= (uint32_t)__bfloat16_as_ushort(lo) << (16 * col);
            if (stage) continue;
            float part = 0.f;
            int pair = 0;
            if (valid) {
                pair = S.ppair[pf + q];
                const size_t o = (size_t)pair * a.I + rb * 8 + g;
                a.h_hi[o] = __bfloat16_as_ushort(hi);
                a.h_lo[o] = __bfloat16_as_ushort(lo);
                part = __bfloat162float(hi) + __bfloat162float(lo);
            }
            part += __shfl_xor_sync(0xffffffffu, part, 4);
            part += __shfl_xor_sync(0xffffffffu, part, 8);
            part += __shfl_xor_sync(0xffffffffu, part, 16);
            if (g == 0 && valid) red_add_f32(a.hsum + (size_t)pair * GI + (rb >> 3), part);
        }
        if (stage) stage[nt * 32 + lane] = make_uint2(his, los);
    }
}

// Writes the staged h of the CTA's gate/up jobs [0, njobs) (global job index g0 + f) and adds
// their group sums; run by all 256 consumer threads.
template <int NT>
__device__ void write_staged_h(const DecodeArgs &a, const DecodeSmem &S, const uint2 *stage, int njobs) {
    const int GI = a.I / kGroup, pg = a.I / 8;
    // one thread per (job, n-tile, t, col): the 8 rows g of that column
    for (int i = threadIdx.x; i < njobs * NT * 8; i += kCW * 32) {
        const int f = i / (NT * 8), nt = (i / 8) % NT, t = (i >> 1) & 3, col = i & 1;
        const int gj = S.g0 + f, u = gj / pg, rb = gj % pg;
        const int pf = S.pfirst[u], nu = S.pfirst[u + 1] - pf;
        const int q = nt * 8 + 2 * t + col;
        if (q >= nu) continue;
        const int pair = S.ppair[pf + q];
        float part = 0.f;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            const uint2 v = stage[(f * NT + nt) * 32 + g * 4 + t];
            const uint16_t hi = (uint16_t)(v.x >> (16 * col)), lo = (uint16_t)(v.y >> (16 * col));
            const size_t o = (size_t)pair * a.I + rb * 8 + g;
            a.h_hi[o] = hi;
            a.h_lo[o] = lo;
            part += bf16_bits_to_float(hi) + bf16_bits_to_float(lo);
        }
        red_add_f32(a.hsum + (size_t)pair * GI + (rb >> 3), part);
    }
}

// ------------------------------------------------------------------------------ top-k
// Every CTA selects the top-k of each token from the logits in L2: stage 1, each (token,
// slice) task keeps the k best of its E/8 experts (warp arg-max rounds); stage 2, each
// candidate's rank among the token's 8k candidates is counted in parallel (larger logit first,
// equal logits -> lower index); stage 3, softmax over the k selected.
__device__ void cta_topk(const DecodeArgs &a, DecodeSmem &S, uint32_t *cand_key, int *cand_idx, int warp, int lane) {
    const int T = a.T, E = a.E, K = a.k;
    const int NC = kSlices * K;                 // candidates per token
    const int slice = (E + kSlices - 1) / kSlices;
    for (int task = warp; task < T * kSlices; task += kWarps) {
        const int t = task / kSlices, sl = task % kSlices;
        const int e0 = sl * slice, e1 = min(E, e0 + slice);
        uint32_t key[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int e = e0 + lane + 32 * m;
            uint32_t kk = 0;
            if (e < e1) {
                float v = __ldcg(a.logits + (size_t)t * E + e);
                if (v != v) v = -INFINITY;
                kk = order_key(v);
            }
            key[m] = kk;
        }
        for (int r = 0; r < K; ++r) {
            uint32_t bk = 0;
            int bm = 0;
#pragma unroll
            for (int m = 0; m < 4; ++m)
                if (key[m] > bk) { bk = key[m]; bm = m; }
            const uint32_t mx = __reduce_max_sync(0xffffffffu, bk);
            const uint32_t cidx = (bk == mx && mx != 0) ? (uint32_t)(e0 + lane + 32 * bm) : 0xFFFFFFFFu;
            const uint32_t win = __reduce_min_sync(0xffffffffu, cidx);
            if (lane == 0) {
                cand_key[t * NC + sl * K + r] = mx;      // 0: slice exhausted
                cand_idx[t * NC + sl * K + r] = (int)win;
            }
            if (mx != 0 && win == (uint32_t)(e0 + lane + 32 * bm)) {
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    if (m == bm) key[m] = 0;
            }
        }
    }
    __syncthreads();
    // stage 2: per token, the k best of its 8k candidates (same order: key desc, index asc)
    for (int t = warp; t < T; t += kWarps) {
        uint32_t ck[8];
        int ci[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int j = lane + 32 * m;
            ck[m] = (j < NC) ? cand_key[t * NC + j] : 0u;
            ci[m] = (j < NC) ? cand_idx[t * NC + j] : 0x7FFFFFFF;
        }
        for (int r = 0; r < K; ++r) {
            uint32_t bk = 0;
            int bi = 0x7FFFFFFF, bm = 0;
#pragma unroll
            for (int m = 0; m < 8; ++m)
                if (ck[m] > bk || (ck[m] == bk && ck[m] != 0 && ci[m] < bi)) { bk = ck[m]; bi = ci[m]; bm = m; }
            const uint32_t mx = __reduce_max_sync(0xffffffffu, bk);
            const uint32_t win = __reduce_min_sync(0xffffffffu, (bk == mx) ? (uint32_t)bi : 0xFFFFFFFFu);
            if (lane == 0) {
                S.sel_idx[t * K + r] = (int)win;
                S.sel_key[t * K + r] = mx;
            }
            if (bk == mx && (uint32_t)bi == win) {
#pragma unroll
                for (int m = 0; m < 8; ++m)
                    if (m == bm) ck[m] = 0;
            }
        }
    }
    __syncthreads();
    for (int t = warp; t < T; t += kWarps) {
        const float v = (lane < K) ? key_value(S.sel_key[t * K + lane]) : -INFINITY;
        const float v0 = __shfl_sync(0xffffffffu, v, 0);
        float ex = 0.f;
        if (lane < K) ex = (v0 == -INFINITY) ? 1.f : expf(v - v0);
        float s = ex;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane < K) {
            const float w = ex / s;
            S.sel_w[t * K + lane] = w;
            if (blockIdx.x == 0 && a.idx_out) a.idx_out[t * K + lane] = S.sel_idx[t * K + lane];
            if (blockIdx.x == 0 && a.w_out) a.w_out[t * K + lane] = w;
        }
    }
}

// ------------------------------------------------------------------------------ kernel
template <int NT>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t dyn[];
    DecodeSmem &S = *reinterpret_cast<DecodeSmem *>(dyn);
    uint8_t *stages = dyn + align_up(sizeof(DecodeSmem), 128);
    uint8_t *act = stages + (size_t)kStages * kStageBytes;
    float *red = reinterpret_cast<float *>(act + kActBytes);
    uint2 *hstage = reinterpret_cast<uint2 *>(act + kActBytes + kRedBytes);
    float *Xs = reinterpret_cast<float *>(act + kActBytes + kRedBytes + kHStageBytes);
    const int T = a.T, H = a.H, I = a.I, E = a.E, K = a.k, P = T * K;
    const int G = H / kGroup, GI = I / kGroup;
    constexpr int NSLOT = 8 / NT;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nC = gridDim.x, c = blockIdx.x;
    uint32_t *status = &a.ctl->status;
    const bool xs_on = x_in_smem(T, H);
    const bool hs_on = h_smem_bytes(P, I) <= (size_t)kActBytes;
    const uint16_t *xsm = xs_on ? reinterpret_cast<const uint16_t *>(act) : nullptr;
    const int ne = (E > c) ? (E - c + nC - 1) / nC : 0;   // router rows of this CTA: c, c+nC, ...
    const bool wr_on = (size_t)ne * H * 4 <= (size_t)kStages * kStageBytes;
    const float *wsm = reinterpret_cast<const float *>(stages);

    // ---------------------------------------------------------------- prologue
    // Reads only the router weights and the packed layer (weights), so it may overlap the
    // previous launch in the stream.
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&S.full[s]), 1);
            mbar_init(smem_u32(&S.empty[s]), kCW);
        }
        mbar_init(smem_u32(&S.wbar), 1);
        mbar_init(smem_u32(&S.xbar), 1);
        fence_barrier_init();
        S.abort = 0;
        S.is_last = 0;
        if (wr_on && ne > 0) {
            const uint32_t rowb = (uint32_t)H * 4;
            mbar_expect_tx(smem_u32(&S.wbar), rowb * ne);
            for (int i = 0; i < ne; ++i)
                bulk_g2s(smem_u32(stages + (size_t)i * rowb), a.wr + (size_t)(c + i * nC) * H, rowb, smem_u32(&S.wbar));
        }
    }
    if (!wr_on)
        for (int i = threadIdx.x; i < ne; i += kThreads) prefetch_l2(a.wr + (size_t)(c + i * nC) * H, (uint32_t)H * 4);
    {
        const PackedExpert *pe = reinterpret_cast<const PackedExpert *>(a.packed + sizeof(PackedHeader));
        for (int e = threadIdx.x; e < E; e += kThreads) {
            const PackedExpert v = pe[e];
            S.eoff[e] = (uint32_t)(v.offset >> 8);
            S.ebits[e] = (uint8_t)v.bits;
        }
    }
    for (int i = threadIdx.x; i < kMaxE / 32; i += kThreads) S.selmask[i] = 0;
    if (threadIdx.x < 8) {
        S.slot_cnt[threadIdx.x] = 0;
        S.slot_seq[threadIdx.x] = 0;
    }
    __syncthreads();
    // Everything below may read data that the previous launch in the stream produces.
    grid_dep_wait();

    // ---------------------------------------------------------------- phase R
    if (xs_on && threadIdx.x == 0) {
        const uint32_t bytes = (uint32_t)(T * H * 2);
        mbar_expect_tx(smem_u32(&S.xbar), bytes);
        bulk_g2s(smem_u32(act), a.x, bytes, smem_u32(&S.xbar));
    }
    const int gtid = c * kThreads + threadIdx.x, gthreads = nC * kThreads;
    for (int i = gtid; i < T * H; i += gthreads) a.out_acc[i] = 0.f;
    for (int i = gtid; i < P * GI; i += gthreads) a.hsum[i] = 0.f;
    if (xs_on && !mbar_wait(smem_u32(&S.xbar), 0, a.wait_ns, status)) S.abort = 1;
    if (wr_on && ne > 0 && !mbar_wait(smem_u32(&S.wbar), 0, a.wait_ns, status)) S.abort = 1;
    const uint16_t *xr = xs_on ? xsm : a.x;
    for (int q = warp; q < ne * T; q += kWarps) {
        const int i = q / T, t = q % T;
        const int e = c + i * nC;
        const float *wrow = wr_on ? wsm + (size_t)i * H : a.wr + (size_t)e * H;
        const uint16_t *xrow = xr + (size_t)t * H;
        float acc = 0.f;
        for (int h = lane * 8; h < H; h += 256) {
            const float4 w0 = *reinterpret_cast<const float4 *>(wrow + h);
            const float4 w1 = *reinterpret_cast<const float4 *>(wrow + h + 4);
            const uint4 xv = *reinterpret_cast<const uint4 *>(xrow + h);
            acc += w0.x * __uint_as_float(xv.x << 16) + w0.y * __uint_as_float(xv.x & 0xFFFF0000u);
            acc += w0.z * __uint_as_float(xv.y << 16) + w0.w * __uint_as_float(xv.y & 0xFFFF0000u);
            acc += w1.x * __uint_as_float(xv.z << 16) + w1.y * __uint_as_float(xv.z & 0xFFFF0000u);
            acc += w1.z * __uint_as_float(xv.w << 16) + w1.w * __uint_as_float(xv.w & 0xFFFF0000u);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) a.logits[(size_t)t * E + e] = acc + (a.bias ? a.bias[e] : 0.f);
    }
    // per-token sums of x over each group (one warp per group, two values per lane)
    for (int i = warp; i < T * G; i += kWarps) {
        const uint32_t v = *reinterpret_cast<const uint32_t *>(xr + (size_t)i * kGroup + 2 * lane);
        float s = __uint_as_float(v << 16) + __uint_as_float(v & 0xFFFF0000u);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) Xs[i] = s;
    }
    __syncthreads();
    if (threadIdx.x == 0 && !grid_barrier(&a.ctl->bar, nC, c == 0, a.wait_ns, status)) S.abort = 1;
    __syncthreads();
    grid_dep_launch();

    // ---------------------------------------------------------------- routing
    const bool aborted = S.abort != 0;
    if (!aborted) {
        uint32_t *cand_key = reinterpret_cast<uint32_t *>(red);
        int *cand_idx = reinterpret_cast<int *>(red) + kSlices * kMaxP;
        cta_topk(a, S, cand_key, cand_idx, warp, lane);
    }
    __syncthreads();
    if (warp == 0 && P <= 32) {
        // unique experts (ascending id), their pair lists (ascending token) and the byte prefixes,
        // one pair per lane
        const bool v = lane < P && !aborted;
        const int e = v ? S.sel_idx[lane] : 0x7FFFFFFF;
        const uint32_t same = __match_any_sync(0xffffffffu, e);
        const bool first = v && (__ffs(same) - 1 == lane);
        int *tmp = reinterpret_cast<int *>(S.cursor);
        tmp[lane] = first ? e : (v ? -1 - e : 0x7FFFFFFF);    // >= 0: first occurrence of an expert
        __syncwarp();
        int slot = 0, before = 0;                             // distinct experts / pairs with a smaller id
#pragma unroll 8
        for (int j = 0; j < 32; ++j) {
            const int ej = tmp[j];
            const int id = ej >= 0 ? ej : -1 - ej;
            if (ej != 0x7FFFFFFF && id < e) {
                ++before;
                slot += ej >= 0 ? 1 : 0;
            }
        }
        const int U = __popc(__ballot_sync(0xffffffffu, first));
        const uint32_t tu = first ? (uint32_t)tile_bytes(S.ebits[e]) / 64 : 0;    // 64-byte units per tile
        if (first) {
            S.ubits[slot] = S.ebits[e];
            S.uoff[slot] = S.eoff[e];
            S.pfirst[slot] = before;
            S.cnt[slot] = __popc(same);
        }
        if (v) {
            const int pos = before + __popc(same & ((1u << lane) - 1u));
            S.ppair[pos] = lane;
            S.ptok[pos] = lane / K;
            S.pw[pos] = S.sel_w[lane];
        }
        __syncwarp();
        // byte prefixes over slots (lane = slot)
        const uint32_t ts = (lane < U) ? (uint32_t)tile_bytes(S.ubits[lane]) / 64 : 0;
        const uint32_t bg = ts * (uint32_t)(I / 8) * G, bd = ts * (uint32_t)(H / 16) * GI;
        uint32_t ig = bg, id = bd;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t og = __shfl_up_sync(0xffffffffu, ig, off);
            const uint32_t od = __shfl_up_sync(0xffffffffu, id, off);
            if (lane >= off) {
                ig += og;
                id += od;
            }
        }
        if (lane < U) {
            S.cgu[lane] = ig - bg;
            S.cd[lane] = id - bd;
        }
        if (lane == U - 1) {
            S.cgu[U] = ig;
            S.cd[U] = id;
        }
        if (lane == 0) {
            S.U = U;
            S.pfirst[U] = aborted ? 0 : P;
            if (U == 0) S.cgu[0] = S.cd[0] = 0;
        }
        (void)tu;
        __syncwarp();
    } else if (warp == 0) {
        // unique experts (ascending id), their pair lists (ascending token) and the byte prefixes
        for (int p = lane; p < (aborted ? 0 : P); p += 32)
            atomicOr(&S.selmask[S.sel_idx[p] >> 5], 1u << (S.sel_idx[p] & 31));
        __syncwarp();
        {
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
        __syncwarp();
        const int U = S.U;
        for (int u = lane; u < U; u += 32) S.cnt[u] = 0;
        __syncwarp();
        for (int p = lane; p < (aborted ? 0 : P); p += 32) {
            const int e = S.sel_idx[p];
            const int u = slot_of(S, e);
            S.ubits[u] = S.ebits[e];
            S.uoff[u] = S.eoff[e];
            atomicAdd(&S.cnt[u], 1);
        }
        __syncwarp();
        int carry = 0;
        uint32_t cg = 0, cdd = 0;
        for (int base = 0; base < U; base += 32) {
            const int u = base + lane;
            const int n = (u < U) ? S.cnt[u] : 0;
            const uint32_t tu = (u < U) ? (uint32_t)tile_bytes(S.ubits[u]) / 64 : 0;   // 64-byte units per tile
            const uint32_t bg = tu * (uint32_t)(I / 8) * G, bd = tu * (uint32_t)(H / 16) * GI;
            int incl = n;
            uint32_t ig = bg, id = bd;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, incl, off);
                const uint32_t og = __shfl_up_sync(0xffffffffu, ig, off);
                const uint32_t od = __shfl_up_sync(0xffffffffu, id, off);
                if (lane >= off) {
                    incl += o;
                    ig += og;
                    id += od;
                }
            }
            if (u < U) {
                S.pfirst[u] = carry + incl - n;
                S.cursor[u] = carry + incl - n;
                S.cgu[u] = cg + ig - bg;
                S.cd[u] = cdd + id - bd;
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
            cg += __shfl_sync(0xffffffffu, ig, 31);
            cdd += __shfl_sync(0xffffffffu, id, 31);
        }
        if (lane == 0) {
            S.pfirst[U] = carry;
            S.cgu[U] = cg;
            S.cd[U] = cdd;
        }
        __syncwarp();
        // stable fill: pairs in ascending pair id (token-major) order
        for (int base = 0; base < (aborted ? 0 : P); base += 32) {
            const int p = base + lane;
            const int u = (p < P) ? slot_of(S, S.sel_idx[p]) : -1 - lane;
            const uint32_t peers = __match_any_sync(0xffffffffu, u);
            const int rank = __popc(peers & ((1u << lane) - 1u));
            if (p < P) {
                const int pos = S.cursor[u] + rank;
                S.ppair[pos] = p;
                S.ptok[pos] = p / K;
                S.pw[pos] = S.sel_w[p];
            }
            __syncwarp();
            if (p < P && rank == 0) S.cursor[u] += __popc(peers);
            __syncwarp();
        }
    }
    if (warp == 0) {
        // Job ranges: the gate/up sequence is cut at multiples of its bytes / nCTA; the down
        // sequence is cut so that each CTA's gate/up + down bytes are the layer's bytes / nCTA.
        // That cut is monotone in the CTA index when every CTA's down share exceeds one gate/up
        // job (plus rounding); otherwise (tiny layers) the down sequence is cut on its own.
        // 32-bit arithmetic: floor(X * c / nC) = (X / nC) * c + ((X % nC) * c) / nC
        __syncwarp();
        const int Uj = aborted ? 0 : S.U;
        const int pg = I / 8, pd = H / 16;
        const uint32_t GUB = S.cgu[Uj], DB = S.cd[Uj], B = GUB + DB;
        auto cut = [&](uint32_t X, int cc) -> uint32_t {
            return (X / nC) * (uint32_t)cc + ((X % nC) * (uint32_t)cc) / nC;
        };
        uint32_t mj = 0;                        // largest gate/up job (64-byte units)
        for (int u = lane; u < Uj; u += 32) mj = max(mj, (S.cgu[u + 1] - S.cgu[u]) / pg);
        mj = __reduce_max_sync(0xffffffffu, mj);
        const bool mono = (uint64_t)(mj + 2) * nC <= DB;
        // lane 0 / 1: the gate/up cut at c / c+1; then lanes 0 / 1: the down cut at c / c+1
        int gcut = 0;
        if (lane < 2) {
            const int cc = c + lane;
            gcut = (cc >= nC) ? Uj * pg : job_at_unit(S.cgu, Uj, pg, cut(GUB, cc));
        }
        const int g0 = __shfl_sync(0xffffffffu, gcut, 0), g1 = __shfl_sync(0xffffffffu, gcut, 1);
        int dcut = 0;
        if (lane < 2) {
            const int cc = c + lane;
            const int gj = lane == 0 ? g0 : g1;
            const uint32_t pos = mono ? cut(B, cc) - job_start_unit(S.cgu, Uj, pg, gj) : cut(DB, cc);
            dcut = (cc >= nC) ? Uj * pd : job_at_unit(S.cd, Uj, pd, pos);
        }
        const int d0 = __shfl_sync(0xffffffffu, dcut, 0), d1 = __shfl_sync(0xffffffffu, dcut, 1);
        if (lane == 0) {
            S.g0 = g0;
            S.g1 = g1;
            S.d0 = d0;
            S.d1 = d1;
            S.nGUc = g1 - g0;
        }
    }
    __syncthreads();

    if (warp == kCW) {
        // ------------------------------------------------------------ producer
        if (lane != 0) return;
        uint32_t cc = 0;
        for (int ph = 0; ph < 2; ++ph) {
            const bool gu = ph == 0;
            const int jend = gu ? S.g1 : S.d1;
            for (int j = gu ? S.g0 : S.d0; j < jend;) {
                const Region r = region_at(S, a, gu, j);
                const int nch = region_chunks(r);
                for (int ch = 0; ch < nch; ++ch) {
                    int c0, m;
                    chunk_range(r, nch, ch, c0, m);
                    const int s = cc % kStages;
                    const uint32_t use = cc / kStages;
                    if (use > 0 && !mbar_wait(smem_u32(&S.empty[s]), (use - 1) & 1u, a.wait_ns, status)) return;
                    const uint32_t bytes = (uint32_t)(m * r.tb);
                    const uint32_t fb = smem_u32(&S.full[s]);
                    mbar_expect_tx(fb, bytes);
                    bulk_g2s(smem_u32(stages + (size_t)s * kStageBytes), r.src + (size_t)c0 * r.tb, bytes, fb);
                    ++cc;
                }
                j += r.tiles / r.tpj;
            }
        }
        return;
    }
    const int nGUc = S.nGUc;
    const bool staged = (size_t)nGUc * NT * 32 * sizeof(uint2) <= (size_t)kHStageBytes;
    if (warp == kCW + 1) {
        // ------------------------------------------------------------ gate/up epilogue
        // Finalises the CTA's gate/up jobs in order as the 8 consumer warps flush their partials,
        // so that no consumer warp stalls on SiLU-GLU and the h write.
        for (int f = 0; f < nGUc; ++f) {
            const int slot = f % NSLOT;
            bool ok = true;
            if (lane == 0 && ld_acquire_cta(&S.slot_cnt[slot]) != kCW) {
                const uint64_t t0 = global_timer();
                while (ld_acquire_cta(&S.slot_cnt[slot]) != kCW) {
                    if (global_timer() - t0 > a.wait_ns) {
                        atomicOr(status, kStatusTimeout);
                        ok = false;
                        break;
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (ok && !aborted) {
                const int gj = S.g0 + f;
                gu_finalize<NT>(a, S, gj / (I / 8), gj % (I / 8), red + (size_t)slot * kCW * NT * 128, lane,
                                staged ? hstage + (size_t)f * NT * 32 : nullptr);
            }
            __syncwarp();
            if (lane == 0) {
                S.slot_cnt[slot] = 0;
                st_release_cta(&S.slot_seq[slot], f / NSLOT + 1);
            }
        }
        gu_done_sync();
        return;
    }

    // ---------------------------------------------------------------- consumers
    uint32_t cc = 0;
    bool skip = aborted;
    const uint8_t *hsm = nullptr;
    int cur = -1, cur_u = 0, cur_rb = 0;   // job in progress (CTA-local index), -1: none
    bool cur_any = false;
    int next_flush = 0;                    // gate/up jobs below this index are flushed by this warp
    bool gu_done = false;
    float acc[NT][4], acc2[NT][4];
    JobCtx<NT> jc;
    const int g = lane >> 2, t = lane & 3;
    auto zero_acc = [&]() {
#pragma unroll
        for (int i = 0; i < NT; ++i) {
            acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
            acc2[i][0] = acc2[i][1] = acc2[i][2] = acc2[i][3] = 0.f;
        }
    };
    auto set_ctx = [&](int u, bool gu) {
        const int pf = S.pfirst[u];
        const int nu = S.pfirst[u + 1] - pf;
        const uint16_t *hh = hsm ? reinterpret_cast<const uint16_t *>(hsm) : a.h_hi;
        const uint16_t *hl = hsm ? reinterpret_cast<const uint16_t *>(hsm) + (size_t)P * I : a.h_lo;
        const float *hs = hsm ? reinterpret_cast<const float *>(hsm + (size_t)2 * P * I * 2) : a.hsum;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int q = nt * 8 + g, q0 = nt * 8 + 2 * t, q1 = q0 + 1;
            if (gu) {
                jc.b[nt] = q < nu ? (xs_on ? xsm : a.x) + (size_t)S.ptok[pf + q] * H : nullptr;
                jc.b2[nt] = nullptr;
                jc.xs0[nt] = q0 < nu ? Xs + (size_t)S.ptok[pf + q0] * G : nullptr;
                jc.xs1[nt] = q1 < nu ? Xs + (size_t)S.ptok[pf + q1] * G : nullptr;
            } else {
                jc.b[nt] = q < nu ? hh + (size_t)S.ppair[pf + q] * I : nullptr;
                jc.b2[nt] = q < nu ? hl + (size_t)S.ppair[pf + q] * I : nullptr;
                jc.xs0[nt] = q0 < nu ? hs + (size_t)S.ppair[pf + q0] * GI : nullptr;
                jc.xs1[nt] = q1 < nu ? hs + (size_t)S.ppair[pf + q1] * GI : nullptr;
            }
        }
    };
    // gate/up: hand this warp's partial of CTA-local job f (acc + acc2, or zeros) to slot
    // f % NSLOT for the epilogue warp. Every warp flushes every job, in order.
    auto gu_flush = [&](int f, bool zeros) {
        const int slot = f % NSLOT;
        const int seq = f / NSLOT;
        if (lane == 0 && ld_acquire_cta(&S.slot_seq[slot]) != seq) {
            const uint64_t t0 = global_timer();
            while (ld_acquire_cta(&S.slot_seq[slot]) != seq) {
                if (global_timer() - t0 > a.wait_ns) {
                    atomicOr(status, kStatusTimeout);
                    break;
                }
            }
        }
        __syncwarp();
        float *rs = red + (size_t)slot * kCW * NT * 128;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
            *reinterpret_cast<float4 *>(rs + ((warp * NT + nt) * 32 + lane) * 4) =
                zeros ? make_float4(0.f, 0.f, 0.f, 0.f)
                      : make_float4(acc[nt][0] + acc2[nt][0], acc[nt][1] + acc2[nt][1], acc[nt][2] + acc2[nt][2],
                                    acc[nt][3] + acc2[nt][3]);
        __syncwarp();
        if (lane == 0) atom_add_acq_rel_cta(&S.slot_cnt[slot], 1);
        __syncwarp();
    };
    auto down_flush = [&]() {
        const int pf = S.pfirst[cur_u];
        const int nu = S.pfirst[cur_u + 1] - pf;
        const int row = cur_rb * 16 + g;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int col = 0; col < 2; ++col) {
                const int q = nt * 8 + 2 * t + col;
                if (q < nu) {
                    const int tok = S.ptok[pf + q];
                    const float wgt = S.pw[pf + q];
                    red_add_f32(a.out_acc + (size_t)tok * H + row, wgt * (acc[nt][col] + acc2[nt][col]));
                    red_add_f32(a.out_acc + (size_t)tok * H + row + 8, wgt * (acc[nt][2 + col] + acc2[nt][2 + col]));
                }
            }
        }
    };
    auto flush_current = [&]() {
        if (cur < 0) return;
        if (cur < nGUc) {
            gu_flush(cur, false);
            next_flush = cur + 1;
        } else if (cur_any && !skip) {
            down_flush();
        }
    };
    auto finish_gu = [&]() {
        if (gu_done) return;
        for (int f = next_flush; f < nGUc; ++f) gu_flush(f, true);
        next_flush = nGUc;
        gu_done = true;
    };
    auto switch_job = [&](int job, int u, int rb, bool gu_job) {
        flush_current();
        if (gu_job) {
            for (int f = next_flush; f < job; ++f) gu_flush(f, true);
            next_flush = job;
        } else {
            finish_gu();
        }
        cur = job;
        cur_u = u;
        cur_rb = rb;
        cur_any = false;
        zero_acc();
        set_ctx(u, gu_job);
    };
    zero_acc();
    for (int ph = 0; ph < 2; ++ph) {
        const bool gu = ph == 0;
        if (!gu) {
            // leaving the gate/up phase: flush the last job and every job this warp skipped
            flush_current();
            cur = -1;
            finish_gu();
            gu_done_sync();
            if (staged && !skip) write_staged_h<NT>(a, S, hstage, nGUc);
            // every h of every CTA is written before any down tile is multiplied
            __threadfence();
            consumer_sync();
            if (threadIdx.x == 0 && !grid_barrier(&a.ctl->bar, nC, c == 0, a.wait_ns, status)) S.abort = 1;
            consumer_sync();
            skip = skip || (S.abort != 0);
            if (hs_on && !skip && S.d1 > S.d0) {
                const size_t hb = (size_t)P * I * 2;
                const size_t sb = align_up((size_t)P * GI * 4, 16);
                const uint4 *s0 = reinterpret_cast<const uint4 *>(a.h_hi);
                const uint4 *s1 = reinterpret_cast<const uint4 *>(a.h_lo);
                const uint4 *s2 = reinterpret_cast<const uint4 *>(a.hsum);
                uint4 *d = reinterpret_cast<uint4 *>(act);
                for (size_t i = threadIdx.x; i < hb / 16; i += kCW * 32) d[i] = __ldcg(s0 + i);
                for (size_t i = threadIdx.x; i < hb / 16; i += kCW * 32) d[hb / 16 + i] = __ldcg(s1 + i);
                for (size_t i = threadIdx.x; i < sb / 16; i += kCW * 32) d[2 * hb / 16 + i] = __ldcg(s2 + i);
                consumer_sync();
                hsm = act;
            }
        }
        const int jend = gu ? S.g1 : S.d1;
        for (int j = gu ? S.g0 : S.d0; j < jend;) {
            const Region r = region_at(S, a, gu, j);
            const int nch = region_chunks(r);
            for (int ch = 0; ch < nch; ++ch) {
                int c0, m;
                chunk_range(r, nch, ch, c0, m);
                const int s = cc % kStages;
                const uint32_t use = cc / kStages;
                if (!mbar_wait(smem_u32(&S.full[s]), use & 1u, a.wait_ns, status)) return;
                const uint8_t *sb = stages + (size_t)s * kStageBytes;
                // this warp's tiles of the chunk: the contiguous block [w0, w1) of region tiles,
                // taken job by job
                const int w0 = c0 + (m * warp) / kCW, w1 = c0 + (m * (warp + 1)) / kCW;
                const int jlo = w0 / r.tpj, jhi = (w1 - 1) / r.tpj;
                for (int jb = jlo; w1 > w0 && jb <= jhi; ++jb) {
                    const int ti0 = max(w0, jb * r.tpj), s1 = min(w1, (jb + 1) * r.tpj);
                    if (ti0 >= s1) continue;
                    const int job = r.job0 + jb;
                    if (job != cur) switch_job(job, r.u, r.rb0 + jb, gu);
                    cur_any = true;
                    if (skip) continue;
                    const int kg0 = ti0 - jb * r.tpj;
                    const uint8_t *tp0 = sb + (size_t)(ti0 - c0) * r.tb;
                    const int ntile = s1 - ti0;                     // this warp's tiles of the job here
#define MOE_RUN(B, GUF)                                                                                   \
    for (int i = 0; i < ntile; i += 2) {                                                                  \
        const bool two = i + 1 < ntile;                                                                   \
        const int i2 = two ? i + 1 : i;                                                                   \
        consume_tile<B, NT, GUF>(tp0 + (size_t)i * r.tb, kg0 + i, jc, lane, acc);                         \
        consume_tile<B, NT, GUF>(tp0 + (size_t)i2 * r.tb, kg0 + i2, jc, lane, acc2, two ? 1.f : 0.f);     \
    }
                    if (gu) {
                        if (r.bits == 4) { MOE_RUN(4, true) }
                        else if (r.bits == 6) { MOE_RUN(6, true) }
                        else { MOE_RUN(8, true) }
                    } else {
                        if (r.bits == 4) { MOE_RUN(4, false) }
                        else if (r.bits == 6) { MOE_RUN(6, false) }
                        else { MOE_RUN(8, false) }
                    }
#undef MOE_RUN
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&S.empty[s]));
                ++cc;
            }
            j += r.tiles / r.tpj;
        }
    }
    flush_current();   // the last down job
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
        const float4 *acc4 = reinterpret_cast<const float4 *>(a.out_acc);
        uint2 *out4 = reinterpret_cast<uint2 *>(a.out);
        for (int i = threadIdx.x; i < T * H / 4; i += kCW * 32) {
            const float4 v = __ldcg(acc4 + i);
            const __nv_bfloat162 lo2 = __floats2bfloat162_rn(v.x, v.y), hi2 = __floats2bfloat162_rn(v.z, v.w);
            out4[i] = make_uint2(*reinterpret_cast<const uint32_t *>(&lo2), *reinterpret_cast<const uint32_t *>(&hi2));
        }
        if (threadIdx.x == 0) a.ctl->done = 0;
    }
}

template <int NT>
moe_status_t launch_nt(const DecodeArgs &a, size_t smem, const DeviceInfo *dev, cudaStream_t st) {
    static bool attr_set[64] = {false};
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d >= 64) return MOE_ERR_CUDA;
    if (!attr_set[d]) {
        if (cudaFuncSetAttribute(decode_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dev->max_smem_optin) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_set[d] = true;
    }
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<NT>, kThreads, smem) != cudaSuccess ||
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
    if (cudaLaunchKernelEx(&cfg, decode_kernel<NT>, a) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

}  // namespace

moe_status_t launch_decode(const uint16_t *x, const float *wr, const float *bias, const void *packed,
                           int T, int H, int I, int E, int k, uint16_t *out, int32_t *idx_out,
                           float *w_out, void *ws, cudaStream_t st) {
    if (T * k > kMaxP) return MOE_ERR_UNSUPPORTED;
    const DeviceInfo *dev = device_info();
    if (!dev) return MOE_ERR_CUDA;
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
    if (T <= 8) return launch_nt<1>(a, smem, dev, st);
    if (T <= 16) return launch_nt<2>(a, smem, dev, st);
    return launch_nt<4>(a, smem, dev, st);
}

}  // namespace moe
