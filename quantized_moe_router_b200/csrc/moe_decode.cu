// moe_decode.cu -- the decode megakernel: one persistent launch per layer computes routing,
// gate/up, SiLU-GLU, down and the weighted combine of the MoE expert block for T <= 32 tokens.
//
// This is the "MoE megakernel" of the page "Raon-1-mini ... RTX 5070 Ti" (table row: one
// persistent kernel for each layer's expert block) with the "pipelined megakernel" row's
// overlap (the next weights are in flight while the current ones are multiplied), laid out for
// sm_100a. One CTA per SM: 16 consumer warps (8 above 16 tokens) and one control warp. Up to 16
// tokens the consumers form two groups of eight warps that take alternate work units, each with
// its own barriers and h buffers, so that one group's barriers and SiLU-GLU overlap the other
// group's multiplications.
//   * Prologue, before the programmatic-dependent-launch wait (it overlaps the previous
//     layer): mbarrier set-up, this CTA's router rows copied into shared memory, the packed
//     layer's expert table read. Both are weights, never produced by the previous launch.
//   * Routing. x is copied into shared memory; each CTA computes the fp32 logits of its
//     E / nCTA experts and publishes each as one 8-byte word {logit, call tag} into up to 32
//     copies of the T x E block, so that the CTAs' polls spread over the L2 slices. Every CTA
//     polls its copy until all words carry this call's tag (derived from a completion counter
//     that grows by nCTA per call: no barrier, no reset) and runs the same top-k + softmax, so
//     all CTAs agree on the selection without a second exchange.
//   * Work units. A unit is (selected expert, 16 consecutive intermediate rows): the unit's
//     gate/up rows (two 8-row blocks over all of H), SiLU-GLU of those 16 rows, and the matching
//     16 columns of the down matrix over all H output rows. Everything a unit needs is on the
//     CTA that runs it, so no intermediate leaves the SM; the units (expert-major) are cut into
//     one contiguous range per CTA with equal bytes.
//   * Streaming. The control warp issues the bulk copies of its range's weights (a unit is three
//     contiguous pieces: gate/up tiles, the down quarter, the down scale/zero entries) into a ring
//     of 48 KB stages as soon as the selection is known; consumers free stages as they go.
//   * Gate/up: tile kg of the unit goes to consumer warp kg % 16 (split K), multiplied with
//     mma.sync on bf16 operands made from the codes by one LOP3 per register (exact integers
//     128 + q), the group's scale and zero applied in fp32; the warps' partial sums meet in shared
//     memory, and one warp per 8 tokens forms h = silu(g) * u as a bf16 hi + lo pair.
//   * Down: super-tile st (64 output rows) of the unit's quarter goes to warp st % 16. One token:
//     w * y is accumulated in shared memory across all of the CTA's units and added into the fp32
//     output accumulator once, four rows per vector reduction. Several tokens: each super-tile's
//     w * y is added into the accumulator as soon as it is computed.
//   * Completion: one counter per 256 output rows; the CTA that completes a row group converts it
//     to bf16 and clears it for the next call.
// Every wait is bounded; on expiry the kernel records MOE_ERR_TIMEOUT in the workspace, the
// warps skip the remaining work in lock step, and the call still leaves the workspace clean.
#include <atomic>

#include "moe_internal.cuh"
#include "moe_topk.cuh"

namespace moe {
namespace {

#ifndef MOE_DECODE_GROUPS
#define MOE_DECODE_GROUPS 2                 // consumer groups up to 16 tokens
#endif
constexpr int kMaxCW = 16;                  // consumer warps at most (+ one control warp)
constexpr int kMaxWarps = kMaxCW + 1;
constexpr int kSlice = 16;                  // intermediate rows per work unit
constexpr int kStageBytes = 49152;          // bytes per ring stage (measured: 24 KB and 32 KB slower)
constexpr int kMaxStages = 8;
constexpr int kActBytes = 65536;            // x of all tokens in shared memory (more: read through L2)
constexpr int kMaxP = kDecodeMaxP;
constexpr int kSmemBudget = 232448;         // 227 KB opt-in shared memory per CTA
constexpr int kBiasRows = 32;               // router bias values kept in shared memory

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
    unsigned long long *logits;
    unsigned long long *rowcnt;
    float *out_acc;
    uint64_t wait_ns;
    uint32_t kmul;               // ceil(2^16 / k): p / k = (p * kmul) >> 16 for p < 2048
    int lrep;                    // copies of the logit words (a power of two)
    int lstride;                 // words between copies
    int lsh, lsl;                // slices per router dot product (2^lsh) and their length
};

// Chunking of one work unit for one code width: gate/up tiles and down super-tiles, each cut into
// nearly equal chunks of at most one ring stage (chunk c of n items: c * base + min(c, rem), with
// base + 1 items for c < rem), and the byte offsets of an expert's parts.
struct WidthPlan {
    int tb, qb;                   // gate/up tile bytes, down super-tile quarter bytes
    int ngc, gbase, grem;         // gate/up chunks of the unit's KG group columns (2 tiles each)
    int ndc, dbase, drem;         // down chunks of its H / 64 super-tiles
    uint32_t gu_part, d_block;    // bytes of the expert's gate/up part, of one down group block
};
__device__ __forceinline__ int width_index(int bits) { return (bits - 4) >> 1; }

struct __align__(16) DecodeSmem {
    WidthPlan wplan[3];
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t xbar, wbar;
    unsigned long long epoch;
    unsigned long long ccost[kMaxP + 1];   // bytes of the units of expert slots < j
    volatile int abort;
    int U, u0, u1;
    uint32_t eoff[kMaxE];               // packed offset / 256 of every expert
    uint8_t ebits[kMaxE];               // code width of every expert
    uint32_t selmask[kMaxE / 32];
    int wordpre[kMaxE / 32];
    int ubits[kMaxP];
    uint32_t uoff[kMaxP];
    int cnt[kMaxP];
    int pfirst[kMaxP + 1];
    int cursor[kMaxP];
    int ptok[kMaxP];
    float pw[kMaxP];
    int sel_idx[kMaxP];
    float sel_w[kMaxP];
    float lpart[4 * kMaxWarps];         // slice sums of the router dot products
    unsigned long long cand[kMaxWarps * 32];   // one token's top-k candidates, k per warp
    unsigned long long selk[kMaxK];     // the selection in order
    float bias[kBiasRows];              // router bias of the CTA's rows c, c + nCTA, ...
};

// Shared-memory regions after DecodeSmem. NT: MMA n-tiles (8 tokens each) of a unit.
struct DecodeLayout {
    size_t xs, xsum, gred, hbuf, hcol, ycta, ring, total;
    int stages;
};
template <int NT, int CW, int NG>
DecodeLayout decode_layout(int T, int H, int smem_limit) {
    DecodeLayout L;
    size_t o = align_up(sizeof(DecodeSmem), 128);
    L.xs = o;
    if ((size_t)T * H * 2 <= (size_t)kActBytes) o += align_up((size_t)T * H * 2, 128);
    L.xsum = o;                                   // x group sums [T x H/64] fp32
    o += align_up((size_t)T * (H / kGroup) * 4, 128);
    L.gred = o;                                   // gate/up partial sums of each warp [CW][2][NT][4][32] fp32
    o += (size_t)CW * 2 * NT * 4 * 32 * 4;
    L.hbuf = o;                                   // per consumer group: h hi / lo [2][NT][8 pairs][16] bf16
    o += (size_t)NG * 2 * NT * 8 * 16 * 2;
    L.hcol = o;                                   // per group: h of each of the 16 rows and pair columns [16][NT x 8] fp32
    o += (size_t)NG * 16 * NT * 8 * 4;
    L.ycta = o;                                   // one token, per group: the CTA's output rows [H] fp32
    if (T == 1) o += (size_t)NG * align_up((size_t)H * 4, 128);
    L.ring = align_up(o, 128);
    const long long room = (long long)min(smem_limit, kSmemBudget) - (long long)L.ring;
    L.stages = room > 0 ? (int)(room / kStageBytes) : 0;
    if (L.stages > kMaxStages) L.stages = kMaxStages;
    L.total = L.ring + (size_t)L.stages * kStageBytes;
    return L;
}

template <int CW>
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(CW * 32) : "memory"); }
// The same barrier, returning the OR of `flag` over the consumer threads: a decision that all
// consumer warps take identically (S.abort can change at any time, so reading it after a plain
// barrier could split the warps).
template <int CW>
__device__ __forceinline__ bool consumer_sync_or(bool flag) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)flag), "n"(CW * 32)
        : "memory");
    return r != 0;
}
// Named barriers 3 and 4: the two consumer groups (NG = 2, CW / 2 warps each); with one group the
// consumer barrier 1.
template <int NG, int CW>
__device__ __forceinline__ void group_sync(int gi) {
    if (NG == 1) consumer_sync<CW>();
    else asm volatile("bar.sync %0, %1;" ::"r"(3 + gi), "n"(CW / NG * 32) : "memory");
}
template <int NG, int CW>
__device__ __forceinline__ bool group_sync_or(int gi, bool flag) {
    if (NG == 1) return consumer_sync_or<CW>(flag);
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)flag), "r"(3 + gi), "n"(CW / NG * 32)
        : "memory");
    return r != 0;
}
// named barrier 2: the control warp arrives when the plan is in shared memory, the consumer
// warps wait for it
template <int CW>
__device__ __forceinline__ void plan_ready_arrive() { asm volatile("bar.arrive 2, %0;" ::"n"((CW + 1) * 32) : "memory"); }
template <int CW>
__device__ __forceinline__ void plan_ready_wait() { asm volatile("bar.sync 2, %0;" ::"n"((CW + 1) * 32) : "memory"); }
__device__ __forceinline__ unsigned long long atom_add_acq_rel_u64(unsigned long long *p, unsigned long long v) {
    unsigned long long old;
    asm volatile("atom.acq_rel.gpu.global.add.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
    return old;
}
__device__ __forceinline__ void red_add_v4_f32(float *p, float4 v) {
    asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
                 : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ float lds32f(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
    return v;
}
// predicated shared-memory store (no branch)
__device__ __forceinline__ void sts_if(bool p, int *addr, int v) {
    asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %0, 0;\n\t@q st.shared.u32 [%1], %2;\n\t}" ::"r"((int)p),
                 "r"(smem_u32(addr)), "r"(v)
                 : "memory");
}

// ------------------------------------------------------------------------------ routing
// Largest key of a lane's M keys and its position; on equal keys the lower position (the lower
// expert index) wins, since a tournament node keeps its left entry unless the right one is larger.
template <int M>
__device__ __forceinline__ void lane_best(const uint32_t (&key)[M], uint32_t &bk, int &bm) {
    uint32_t k2[M];
    int m2[M];
#pragma unroll
    for (int i = 0; i < M; ++i) {
        k2[i] = key[i];
        m2[i] = i;
    }
#pragma unroll
    for (int w = 1; w < M; w <<= 1)
#pragma unroll
        for (int i = 0; i + w < M; i += 2 * w)
            if (k2[i + w] > k2[i]) {
                k2[i] = k2[i + w];
                m2[i] = m2[i + w];
            }
    bk = k2[0];
    bm = m2[0];
}

// One comparator of a descending sort of (key, position) pairs: equal keys keep the lower
// position (the lower expert index) first.
// Written with selects: a divergent branch per comparator costs far more than the swap.
__device__ __forceinline__ void sort_ce(uint32_t &ki, int &mi, uint32_t &kj, int &mj) {
    const bool sw = (kj > ki) | ((kj == ki) & (mj < mi));
    const uint32_t k0 = sw ? kj : ki, k1 = sw ? ki : kj;
    const int m0 = sw ? mj : mi, m1 = sw ? mi : mj;
    ki = k0;
    kj = k1;
    mi = m0;
    mj = m1;
}

// Polls token t's exchanged logit words (M per lane: expert lane + 32 m) until every word
// carries `tag`, as order keys (0 where absent; NaN as -inf). False (warp-uniformly) when the
// wait expires.
template <int M>
__device__ __forceinline__ bool poll_keys(const DecodeArgs &a, int t, uint32_t tag, int lane, uint32_t (&key)[M]) {
    const unsigned long long *row =
        a.logits + (size_t)(blockIdx.x & (unsigned)(a.lrep - 1)) * a.lstride + (size_t)t * a.E;
    uint64_t t0 = 0;
    for (int it = 0;; ++it) {
        bool ok = true;
#pragma unroll
        for (int m = 0; m < M; ++m) {
            const int e = lane + 32 * m;
            uint32_t kk = 0;
            if (e < a.E) {
                const unsigned long long v = ld_relaxed_u64(row + e);
                ok = ok && (uint32_t)(v >> 32) == tag;
                float x = __uint_as_float((uint32_t)v);
                if (x != x) x = -INFINITY;
                kk = order_key(x);   // never 0 for a non-NaN value
            }
            key[m] = kk;
        }
        if (__all_sync(0xffffffffu, ok)) return true;
        int expired = 0;
        if (lane == 0) {
            const uint64_t now = global_timer();
            if (it == 0) t0 = now;
            expired = (now - t0 > a.wait_ns) ? 1 : 0;
            if (expired) atomicOr(&a.ctl->status, kStatusTimeout);
        }
        if (__shfl_sync(0xffffffffu, expired, 0)) return false;
        __nanosleep(32);
    }
}

// The softmax weights of a selection, from the rounds' maxima in round order (every lane sees
// them all): lane r < k keeps exp(l_r - l_0), and the sum runs over the rounds in order.
struct SoftmaxAcc {
    float v0 = 0.f, s = 0.f, my_e = 0.f;
    __device__ __forceinline__ void add(uint32_t mx, int r, int lane) {
        const float v = key_value(mx);
        v0 = (r == 0) ? v : v0;
        const float ex = (v0 == -INFINITY) ? 1.f : expf(v - v0);
        s += ex;
        my_e = (lane == r) ? ex : my_e;
    }
};
__device__ __forceinline__ void store_weights(const DecodeArgs &a, DecodeSmem &S, int t, int lane, int c,
                                              const SoftmaxAcc &sm) {
    if (lane < a.k) {
        const float w = sm.my_e / sm.s;
        S.sel_w[t * a.k + lane] = w;
        if (c == 0 && a.w_out) a.w_out[t * a.k + lane] = w;
    }
}

// Exact selection (larger logit first, equal logits -> lower index) of token t, up to 1024
// experts: each round the maximum key, then the lowest index holding it; the winning lane
// rescans its keys. Out of line: it serves wide expert counts and ties of the fast selection.
__device__ __noinline__ bool token_topk_wide(const DecodeArgs &a, DecodeSmem &S, int t, uint32_t tag, int lane, int c) {
    uint32_t key[32];
    if (!poll_keys<32>(a, t, tag, lane, key)) return false;
    const int K = a.k;
    SoftmaxAcc sm;
    uint32_t bk;
    int bm;
    lane_best<32>(key, bk, bm);
    for (int r = 0; r < K; ++r) {
        const uint32_t mx = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t win = __reduce_min_sync(0xffffffffu, bk == mx ? (uint32_t)(lane + 32 * bm) : 0xFFFFFFFFu);
        if (lane == r) {
            S.sel_idx[t * K + r] = (int)win;
            if (c == 0 && a.idx_out) a.idx_out[t * K + r] = (int)win;
        }
        if ((int)(win & 31u) == lane) {
#pragma unroll
            for (int m = 0; m < 32; ++m)
                if (m == bm) key[m] = 0;
            lane_best<32>(key, bk, bm);
        }
        sm.add(mx, r, lane);
    }
    store_weights(a, S, t, lane, c, sm);
    return true;
}

// Top-k of token t (E <= 256: 8 keys per lane), written to S.sel_idx / S.sel_w[t * k + i] (and
// idx_out / w_out from CTA 0); false (warp-uniformly) when the wait for the logits expires.
// Each lane sorts its keys once (equal keys: lower index first); a round takes the maximum of
// the lanes' heads and the lane holding it pops its head, a register shift. When two lanes hold
// that maximum the exact routine redoes the selection.
__device__ bool token_topk(const DecodeArgs &a, DecodeSmem &S, int t, uint32_t tag, int lane, int c) {
    uint32_t sk[8];
    if (!poll_keys<8>(a, t, tag, lane, sk)) return false;
    int sm_[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) sm_[m] = m;
    sort_ce(sk[0], sm_[0], sk[2], sm_[2]); sort_ce(sk[1], sm_[1], sk[3], sm_[3]);
    sort_ce(sk[4], sm_[4], sk[6], sm_[6]); sort_ce(sk[5], sm_[5], sk[7], sm_[7]);
    sort_ce(sk[0], sm_[0], sk[4], sm_[4]); sort_ce(sk[1], sm_[1], sk[5], sm_[5]);
    sort_ce(sk[2], sm_[2], sk[6], sm_[6]); sort_ce(sk[3], sm_[3], sk[7], sm_[7]);
    sort_ce(sk[0], sm_[0], sk[1], sm_[1]); sort_ce(sk[2], sm_[2], sk[3], sm_[3]);
    sort_ce(sk[4], sm_[4], sk[5], sm_[5]); sort_ce(sk[6], sm_[6], sk[7], sm_[7]);
    sort_ce(sk[2], sm_[2], sk[4], sm_[4]); sort_ce(sk[3], sm_[3], sk[5], sm_[5]);
    sort_ce(sk[1], sm_[1], sk[4], sm_[4]); sort_ce(sk[3], sm_[3], sk[6], sm_[6]);
    sort_ce(sk[1], sm_[1], sk[2], sm_[2]); sort_ce(sk[3], sm_[3], sk[4], sm_[4]);
    sort_ce(sk[5], sm_[5], sk[6], sm_[6]);
    const int K = a.k;
    SoftmaxAcc sm;
    uint32_t tied = 0;
    int *sel = S.sel_idx + t * K;
    for (int r = 0; r < K; ++r) {
        const uint32_t mx = __reduce_max_sync(0xffffffffu, sk[0]);
        const bool win = sk[0] == mx;
        const uint32_t b = __ballot_sync(0xffffffffu, win);
        tied |= b & (b - 1u);
        sts_if(win, sel + r, lane + 32 * sm_[0]);
        // the winner shifts its list (selects, no branch)
#pragma unroll
        for (int m = 0; m < 7; ++m) {
            sk[m] = win ? sk[m + 1] : sk[m];
            sm_[m] = win ? sm_[m + 1] : sm_[m];
        }
        sk[7] = win ? 0u : sk[7];
        sm.add(mx, r, lane);
    }
    if (tied) return token_topk_wide(a, S, t, tag, lane, c);
    __syncwarp();
    if (c == 0 && a.idx_out && lane < K) a.idx_out[t * K + lane] = sel[lane];
    store_weights(a, S, t, lane, c, sm);
    return true;
}


// ------------------------------------------------------------------------------ plan
__device__ __forceinline__ int slot_of(const DecodeSmem &S, int e) {
    const int w = e >> 5;
    return S.wordpre[w] + __popc(S.selmask[w] & ((1u << (e & 31)) - 1u));
}

// Expert slots of one token (P = k <= 32 pairs, distinct experts): slot j is selection j.
__device__ __forceinline__ void plan_single(DecodeSmem &S, int P, int lane, bool weights) {
    if (lane < P) {
        const int e = S.sel_idx[lane];
        S.ubits[lane] = S.ebits[e];
        S.uoff[lane] = S.eoff[e];
        S.pfirst[lane] = lane;
        S.ptok[lane] = 0;
        if (weights) S.pw[lane] = S.sel_w[lane];
    }
    if (lane == 0) {
        S.U = P;
        S.pfirst[P] = P;
    }
    __syncwarp();
}

// Expert slots of several tokens, by one warp: the distinct selected experts in ascending id,
// each with its pairs in ascending pair id (token-major, so ascending token).
__device__ __noinline__ void plan_many(const DecodeArgs &a, DecodeSmem &S, int P, int lane) {
    const int E = a.E;
    for (int i = lane; i < kMaxE / 32; i += 32) S.selmask[i] = 0;
    __syncwarp();
    for (int p = lane; p < P; p += 32) atomicOr(&S.selmask[S.sel_idx[p] >> 5], 1u << (S.sel_idx[p] & 31));
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
    for (int p = lane; p < P; p += 32) {
        const int e = S.sel_idx[p];
        const int u = slot_of(S, e);
        S.ubits[u] = S.ebits[e];
        S.uoff[u] = S.eoff[e];
        atomicAdd(&S.cnt[u], 1);
    }
    __syncwarp();
    int carry = 0;
    for (int base = 0; base < U; base += 32) {
        const int u = base + lane;
        const int n = (u < U) ? S.cnt[u] : 0;
        int incl = n;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
        }
        if (u < U) {
            S.pfirst[u] = carry + incl - n;
            S.cursor[u] = carry + incl - n;
        }
        carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) S.pfirst[U] = carry;
    __syncwarp();
    // stable fill: pairs in ascending pair id order
    for (int base = 0; base < P; base += 32) {
        const int p = base + lane;
        const int u = (p < P) ? slot_of(S, S.sel_idx[p]) : -1 - lane;
        const uint32_t peers = __match_any_sync(0xffffffffu, u);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        if (p < P) {
            const int pos = S.cursor[u] + rank;
            S.ptok[pos] = (int)(((uint32_t)p * a.kmul) >> 16);
            S.pw[pos] = S.sel_w[p];
        }
        __syncwarp();
        if (p < P && rank == 0) S.cursor[u] += __popc(peers);
        __syncwarp();
    }
}

// Bytes one work unit of an expert of width `bits` streams: its two gate/up row blocks, its down
// quarter and the down scale/zero entries of its group column.
__device__ __forceinline__ unsigned long long unit_bytes(const DecodeArgs &a, int bits) {
    return (unsigned long long)(2 * (a.H / kGroup)) * tile_bytes(bits) +
           (unsigned long long)(a.H / 64) * d_quarter_bytes(bits) + 4ull * a.H;
}

// 64-bit compare-exchange of a descending sequence: the larger value first
__device__ __forceinline__ void ce64(unsigned long long &a, unsigned long long &b) {
    const unsigned long long hi = a > b ? a : b, lo = a > b ? b : a;
    a = hi;
    b = lo;
}
// Top-k of token t for E <= 256 and k <= 8, by merging: every lane sorts its 8 keys (expert
// lane + 32 m), then five butterfly steps each keep the 8 largest of two lanes' lists (the
// element-wise maximum of one list and the other reversed is a bitonic sequence holding them,
// sorted by a 3-stage network), after which every lane holds the selection in order. Keys are
// 64-bit {order key of the logit, 2^32 - 1 - expert}, so equal logits put the lower expert
// first exactly. The softmax terms are formed one per lane. Writes as token_topk.
__device__ bool token_topk_merge(const DecodeArgs &a, DecodeSmem &S, int t, uint32_t tag, int lane, int c) {
    uint32_t sk[8];
    if (!poll_keys<8>(a, t, tag, lane, sk)) return false;
    int sm_[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) sm_[m] = m;
    sort_ce(sk[0], sm_[0], sk[2], sm_[2]); sort_ce(sk[1], sm_[1], sk[3], sm_[3]);
    sort_ce(sk[4], sm_[4], sk[6], sm_[6]); sort_ce(sk[5], sm_[5], sk[7], sm_[7]);
    sort_ce(sk[0], sm_[0], sk[4], sm_[4]); sort_ce(sk[1], sm_[1], sk[5], sm_[5]);
    sort_ce(sk[2], sm_[2], sk[6], sm_[6]); sort_ce(sk[3], sm_[3], sk[7], sm_[7]);
    sort_ce(sk[0], sm_[0], sk[1], sm_[1]); sort_ce(sk[2], sm_[2], sk[3], sm_[3]);
    sort_ce(sk[4], sm_[4], sk[5], sm_[5]); sort_ce(sk[6], sm_[6], sk[7], sm_[7]);
    sort_ce(sk[2], sm_[2], sk[4], sm_[4]); sort_ce(sk[3], sm_[3], sk[5], sm_[5]);
    sort_ce(sk[1], sm_[1], sk[4], sm_[4]); sort_ce(sk[3], sm_[3], sk[6], sm_[6]);
    sort_ce(sk[1], sm_[1], sk[2], sm_[2]); sort_ce(sk[3], sm_[3], sk[4], sm_[4]);
    sort_ce(sk[5], sm_[5], sk[6], sm_[6]);
    unsigned long long v[8];
#pragma unroll
    for (int m = 0; m < 8; ++m)
        v[m] = sk[m] ? ((unsigned long long)sk[m] << 32) | (0xFFFFFFFFu - (uint32_t)(lane + 32 * sm_[m])) : 0ull;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        unsigned long long o[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) o[m] = __shfl_xor_sync(0xffffffffu, v[m], d);
#pragma unroll
        for (int m = 0; m < 8; ++m) v[m] = v[m] > o[7 - m] ? v[m] : o[7 - m];
        ce64(v[0], v[4]); ce64(v[1], v[5]); ce64(v[2], v[6]); ce64(v[3], v[7]);
        ce64(v[0], v[2]); ce64(v[1], v[3]); ce64(v[4], v[6]); ce64(v[5], v[7]);
        ce64(v[0], v[1]); ce64(v[2], v[3]); ce64(v[4], v[5]); ce64(v[6], v[7]);
    }
    const int K = a.k;
    unsigned long long mine = v[0];
#pragma unroll
    for (int m = 1; m < 8; ++m) mine = (lane == m) ? v[m] : mine;
    const float v0 = key_value((uint32_t)(v[0] >> 32));
    const float my_v = key_value((uint32_t)(mine >> 32));
    float ex = 0.f;
    if (lane < K) ex = (v0 == -INFINITY) ? 1.f : expf(my_v - v0);
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < K) {
        const int e = (int)(0xFFFFFFFFu - (uint32_t)mine);
        const float w = ex / sum;
        S.sel_idx[t * K + lane] = e;
        S.sel_w[t * K + lane] = w;
        if (c == 0 && a.idx_out) a.idx_out[t * K + lane] = e;
        if (c == 0 && a.w_out) a.w_out[t * K + lane] = w;
    }
    __syncwarp();
    return true;
}

// One token's top-k by the whole CTA (E <= 32 x warps, k <= 32). Warp w polls the logits of
// experts 32w .. 32w + 31 (one per lane) and sorts them by a bitonic network across the lanes;
// its k largest become candidates. After a CTA barrier every warp ranks some candidates against
// all of them (ballots); candidate of rank r < k is the r-th selection. Keys are 64-bit {order
// key of the logit, 2^32 - 1 - expert}: equal logits put the lower expert first, exactly.
// Phase 1 (warps w < ceil(E / 32)); returns false (warp-uniformly) when the wait expires.
__device__ __forceinline__ bool topk_one_candidates(const DecodeArgs &a, DecodeSmem &S, uint32_t tag, int warp,
                                                    int lane) {
    const int e = 32 * warp + lane;
    const unsigned long long *row = a.logits + (size_t)(blockIdx.x & (unsigned)(a.lrep - 1)) * a.lstride;
    unsigned long long v = 0ull;
    uint64_t t0 = 0;
    for (int it = 0;; ++it) {
        bool ok = true;
        uint32_t kk = 0;
        if (e < a.E) {
            const unsigned long long w = ld_relaxed_u64(row + e);
            ok = (uint32_t)(w >> 32) == tag;
            float x = __uint_as_float((uint32_t)w);
            if (x != x) x = -INFINITY;
            kk = order_key(x);   // never 0 for a non-NaN value
        }
        if (__all_sync(0xffffffffu, ok)) {
            v = e < a.E ? ((unsigned long long)kk << 32) | (0xFFFFFFFFu - (uint32_t)e) : 0ull;
            break;
        }
        int expired = 0;
        if (lane == 0) {
            const uint64_t now = global_timer();
            if (it == 0) t0 = now;
            expired = (now - t0 > a.wait_ns) ? 1 : 0;
            if (expired) atomicOr(&a.ctl->status, kStatusTimeout);
        }
        if (__shfl_sync(0xffffffffu, expired, 0)) return false;
        __nanosleep(32);
    }
    // bitonic sort across the lanes, descending (lane 0 the largest)
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, stride);
            const bool keep_max = ((lane & stride) == 0) == ((lane & size) == 0);
            v = keep_max ? (v > o ? v : o) : (v > o ? o : v);
        }
    if (lane < a.k) S.cand[warp * a.k + lane] = v;
    return true;
}
// Phase 2 (all threads, after a barrier): thread i ranks candidate i among the C = nw * k
// candidates, four independent counts over all of them.
__device__ __forceinline__ void topk_one_rank(const DecodeArgs &a, DecodeSmem &S, int nw) {
    const int C = nw * a.k, i = threadIdx.x;
    if (i >= C) return;
    const unsigned long long x = S.cand[i];
    int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
    int j = 0;
    for (; j + 4 <= C; j += 4) {
        r0 += S.cand[j] > x;
        r1 += S.cand[j + 1] > x;
        r2 += S.cand[j + 2] > x;
        r3 += S.cand[j + 3] > x;
    }
    for (; j < C; ++j) r0 += S.cand[j] > x;
    const int rank = (r0 + r1) + (r2 + r3);
    if (rank < a.k) S.selk[rank] = x;
}
// Phase 3 (one warp, after a barrier): indices and softmax weights of the selection.
// The selection in order from the ranked keys (the control warp), before the weights.
__device__ __forceinline__ void topk_one_select(const DecodeArgs &a, DecodeSmem &S, int lane) {
    if (lane < a.k) S.sel_idx[lane] = (int)(0xFFFFFFFFu - (uint32_t)S.selk[lane]);
    __syncwarp();
}
// The softmax weights of the selection (also the slots' pair weights; idx_out / w_out from CTA 0).
__device__ __forceinline__ void topk_one_finish(const DecodeArgs &a, DecodeSmem &S, int lane, int c) {
    const int K = a.k;
    const unsigned long long mine = lane < K ? S.selk[lane] : 0ull;
    const float v0 = key_value((uint32_t)(S.selk[0] >> 32));
    const float my_v = key_value((uint32_t)(mine >> 32));
    float ex = 0.f;
    if (lane < K) ex = (v0 == -INFINITY) ? 1.f : expf(my_v - v0);
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < K) {
        const int e = (int)(0xFFFFFFFFu - (uint32_t)mine);
        const float w = ex / sum;
        S.sel_w[lane] = w;
        S.pw[lane] = w;
        if (c == 0 && a.idx_out) a.idx_out[lane] = e;
        if (c == 0 && a.w_out) a.w_out[lane] = w;
    }
    __syncwarp();
}

// floor(n / d) for n < 2^53 through the double quotient (within one of the result), corrected
__device__ __forceinline__ unsigned long long div_floor(unsigned long long n, unsigned long long d) {
    unsigned long long q = (unsigned long long)((double)n / (double)d);
    if (q * d > n) --q;
    if ((q + 1) * d <= n) ++q;
    return q;
}

// This CTA's range of work units [u0, u1): units are numbered slot-major (I / 16 per slot); CTA c
// takes the units whose first byte lies in [c * B / nC, (c + 1) * B / nC) of the B bytes of all.
__device__ void plan_units(const DecodeArgs &a, DecodeSmem &S, int lane, int c, int nC) {
    const int U = S.U, sp = a.I / kSlice;
    {
        // all slots of one width (the usual case): equal units, a 32-bit cut
        bool same = true;
        for (int j = lane; j < U; j += 32) same = same && S.ubits[j] == S.ubits[0];
        if (__all_sync(0xffffffffu, same)) {
            const uint32_t N = (uint32_t)(U * sp);
            if (lane == 0) {
                S.u0 = (int)((uint32_t)c * N / (uint32_t)nC);
                S.u1 = (int)((uint32_t)(c + 1) * N / (uint32_t)nC);
            }
            __syncwarp();
            return;
        }
    }
    unsigned long long carry = 0;
    for (int base = 0; base < U; base += 32) {
        const int j = base + lane;
        const unsigned long long cj = j < U ? (unsigned long long)sp * unit_bytes(a, S.ubits[j]) : 0ull;
        unsigned long long incl = cj;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const unsigned long long o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
        }
        if (j < U) S.ccost[j] = carry + incl - cj;
        carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) S.ccost[U] = carry;
    __syncwarp();
    const unsigned long long B = carry;
    auto unit_at = [&](unsigned long long pos) -> int {
        if (pos >= B) return U * sp;
        int jj = 0;
        for (int base = 0; base < U; base += 32) {
            const int j = base + lane;
            const bool h = j < U && S.ccost[j] <= pos && pos < S.ccost[j + 1];
            const uint32_t m = __ballot_sync(0xffffffffu, h);
            if (m) {
                jj = base + __ffs(m) - 1;
                break;
            }
        }
        const unsigned long long ub = unit_bytes(a, S.ubits[jj]);
        return jj * sp + (int)div_floor(pos - S.ccost[jj] + ub - 1, ub);
    };
    const int u0 = unit_at(div_floor(B * (unsigned long long)c, (unsigned long long)nC));
    const int u1 = (c + 1 >= nC) ? U * sp : unit_at(div_floor(B * (unsigned long long)(c + 1), (unsigned long long)nC));
    if (lane == 0) {
        S.u0 = u0;
        S.u1 = u1;
    }
    __syncwarp();
}

// ------------------------------------------------------------------------------ work units
__device__ __forceinline__ WidthPlan make_width_plan(int H, int I, int bits) {
    WidthPlan w;
    const int KG = H / kGroup, nst = H / 64;
    w.tb = tile_bytes(bits);
    w.qb = d_quarter_bytes(bits);
    const int gcap = kStageBytes / (2 * w.tb), dcap = kStageBytes / (256 + w.qb);
    w.ngc = (KG + gcap - 1) / gcap;
    w.gbase = KG / w.ngc;
    w.grem = KG - w.gbase * w.ngc;
    w.ndc = (nst + dcap - 1) / dcap;
    w.dbase = nst / w.ndc;
    w.drem = nst - w.dbase * w.ndc;
    w.gu_part = (uint32_t)(gu_tiles(H, I) * w.tb);
    w.d_block = (uint32_t)d_block_bytes(H, bits);
    return w;
}
// items [b, e) of chunk c: n = base * parts + rem items cut as above
__device__ __forceinline__ void chunk_items(int base, int rem, int c, int &b, int &e) {
    b = c * base + (c < rem ? c : rem);
    e = b + base + (c < rem ? 1 : 0);
}
// the three pieces of unit (slot j, slice i): gate/up tiles, down scale/zero entries, down quarter
struct UnitGeo {
    const uint8_t *gu, *sz, *q;
};
__device__ __forceinline__ UnitGeo unit_geo(const DecodeArgs &a, const DecodeSmem &S, const WidthPlan &w, int j, int i) {
    UnitGeo g;
    const uint8_t *base = a.packed + (size_t)S.uoff[j] * 256;
    g.gu = base + (size_t)(2 * i) * (a.H / kGroup) * w.tb;
    g.sz = base + w.gu_part + (size_t)(i >> 2) * w.d_block;
    g.q = g.sz + (size_t)4 * a.H + (size_t)(i & 3) * (a.H / 64) * w.qb;
    return g;
}

// ------------------------------------------------------------------------------ tile math
// Operand sources of the current expert slot for this lane: per n-tile, the x row that the
// lane's B column reads (a valid row also where the column has no token: those columns are
// never used) and the group-sum rows of its two accumulator columns.
template <int NT>
struct GuCtx {
    const uint16_t *b[NT];   // global x rows (!xs_on)
    uint32_t sb[NT];         // shared-memory x rows (xs_on)
    uint32_t xs0[NT], xs1[NT];
    bool bg;
};

// D = A * B + D (m16n8k16, bf16 operands, fp32 accumulators). Not volatile: independent MMAs of
// a warp may be scheduled back to back (each has a latency of about 90 cycles on this part).
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 16x64 gate/up tile against one n-tile: the group's four MMAs into four separate
// accumulators (no MMA waits for another), then the group's affine correction
// out += s * (sum - (off + z) * X) with X the group sums of the lane's two accumulator columns.
template <int BITS, bool ONE>
__device__ __forceinline__ void gu_group_mma(const uint4 &lo, const uint4 &hi8, const uint2 &hi6,
                                             const uint32_t (&b)[8], float sA, float zA, float sB, float zB,
                                             float X0, float X1, float (&out)[4]) {
    float c[4][4];
    const uint32_t low[4] = {lo.x, lo.y, lo.z, lo.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        c[j][0] = c[j][1] = c[j][2] = c[j][3] = 0.f;
        const uint32_t w = low[j];
        mma16816(c[j], code_pair<0x000F000Fu>(w, 0), code_pair<0x000F000Fu>(w, 4), code_pair<0x000F000Fu>(w, 8),
                 code_pair<0x000F000Fu>(w, 12), b[2 * j], b[2 * j + 1]);
    }
    if (BITS != 4) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t b0 = bf16x2_mul16(b[2 * j]), b1 = bf16x2_mul16(b[2 * j + 1]);
            if (BITS == 8) {
                const uint32_t w = (j == 0) ? hi8.x : (j == 1) ? hi8.y : (j == 2) ? hi8.z : hi8.w;
                mma16816(c[j], code_pair<0x000F000Fu>(w, 0), code_pair<0x000F000Fu>(w, 4),
                         code_pair<0x000F000Fu>(w, 8), code_pair<0x000F000Fu>(w, 12), b0, b1);
            } else {
                const uint32_t w = (j < 2) ? hi6.x : hi6.y;
                const int s0 = (j & 1) * 8;
                mma16816(c[j], code_pair<0x00030003u>(w, s0 + 0), code_pair<0x00030003u>(w, s0 + 2),
                         code_pair<0x00030003u>(w, s0 + 4), code_pair<0x00030003u>(w, s0 + 6), b0, b1);
            }
        }
    }
    const float off = (BITS == 4) ? 128.f : 2176.f;   // 128 per plane, the hi plane weighted 16x
    const float s0 = (c[0][0] + c[1][0]) + (c[2][0] + c[3][0]), s2 = (c[0][2] + c[1][2]) + (c[2][2] + c[3][2]);
    out[0] += sA * (s0 - (off + zA) * X0);
    out[2] += sB * (s2 - (off + zB) * X0);
    if (!ONE) {   // one token: accumulator column 1 holds no pair
        const float s1 = (c[0][1] + c[1][1]) + (c[2][1] + c[3][1]), s3 = (c[0][3] + c[1][3]) + (c[2][3] + c[3][3]);
        out[1] += sA * (s1 - (off + zA) * X1);
        out[3] += sB * (s3 - (off + zB) * X1);
    }
}

// The two tiles of one group column kg (row blocks 2i and 2i + 1 of the unit, adjacent in the
// packed layer) against the same n-tile operands: the x rows and group sums are read once, and the
// tiles' eight MMAs are independent of each other.
template <int BITS, int NT, bool ONE>
__device__ __forceinline__ void gu_pair(const uint8_t *tile, int kg, const GuCtx<NT> &jc, int lane,
                                        float (&acc)[2][NT][4]) {
    constexpr int tb = tile_bytes(BITS);
    const int g = lane >> 2, t = lane & 3;
    uint4 lo[2], hi8[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
    uint2 hi6[2] = {make_uint2(0, 0), make_uint2(0, 0)};
    float sA[2], zA[2], sB[2], zB[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const uint8_t *tp = tile + r * tb;
        lo[r] = *reinterpret_cast<const uint4 *>(tp + 16 * lane);
        if (BITS == 8) hi8[r] = *reinterpret_cast<const uint4 *>(tp + kLoBytes + 16 * lane);
        if (BITS == 6) hi6[r] = *reinterpret_cast<const uint2 *>(tp + kLoBytes + 8 * lane);
        const uint2 sz = *reinterpret_cast<const uint2 *>(tp + kLoBytes + hi_bytes(BITS) + 8 * g);
        sA[r] = half_lo(sz.x);
        zA[r] = half_hi(sz.x);
        sB[r] = half_lo(sz.y);
        zB[r] = half_hi(sz.y);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        uint4 v0, v1;
        if (jc.bg) {
            const uint4 *p = reinterpret_cast<const uint4 *>(jc.b[nt] + kg * kGroup + 16 * t);
            v0 = __ldcg(p);
            v1 = __ldcg(p + 1);
        } else {
            const uint32_t o = (uint32_t)(kg * kGroup + 16 * t) * 2;
            v0 = lds128(jc.sb[nt] + o);
            v1 = lds128(jc.sb[nt] + o + 16);
        }
        const uint32_t b[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        const float X0 = lds32f(jc.xs0[nt] + kg * 4), X1 = ONE ? 0.f : lds32f(jc.xs1[nt] + kg * 4);
#pragma unroll
        for (int r = 0; r < 2; ++r)
            gu_group_mma<BITS, ONE>(lo[r], hi8[r], hi6[r], b, sA[r], zA[r], sB[r], zB[r], X0, X1, acc[r][nt]);
    }
}

// The warp's gate/up work in a chunk holding the unit's group columns [k0, k1) (two tiles each):
// group column kg goes to warp kg % CW.
template <int BITS, int NT, int CW, bool ONE>
__device__ __forceinline__ void gu_chunk(const uint8_t *stage, int k0, int k1, int warp, const GuCtx<NT> &jc,
                                         int lane, float (&acc)[2][NT][4]) {
    constexpr int tb = tile_bytes(BITS);
    for (int kg = k0 + ((warp - k0) % CW + CW) % CW; kg < k1; kg += CW)
        gu_pair<BITS, NT, ONE>(stage + (size_t)(kg - k0) * 2 * tb, kg, jc, lane, acc);
}

// Down operands of the current unit for this lane: h of the unit's 16 rows for the lane's B
// column (pair g of each n-tile) as bf16 hi / lo pairs (and x16 copies for the 6/8-bit high code
// planes), the sums X of h over the 16 rows and the routing weights of its two accumulator
// columns (0 where the column has no pair).
template <int NT>
struct DnCtx {
    uint32_t hb[NT][2], lb[NT][2], hb16[NT][2], lb16[NT][2];
    float X0[NT], X1[NT], w0[NT], w1[NT];
};

// One 64-row super-tile of the unit's down quarter: four 16x16 MMAs (per n-tile and h half), the
// row's scale and zero and the column's weight applied in fp32: acc += w * s * (sum - (off + z) X).
template <int BITS, int NT, bool ONE>
__device__ __forceinline__ void down_st(uint32_t szp, uint32_t qp, const DnCtx<NT> &dc, int lane,
                                        float (&acc)[4][NT][4]) {
    const int g = lane >> 2;
    float c[4][NT][4], d[4][NT][4];
    // the MMAs of all four 16-row blocks, each into its own accumulators
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const uint32_t w = lds32(qp + r * 128 + 4 * lane);
        const uint32_t a0 = code_pair<0x000F000Fu>(w, 0), a1 = code_pair<0x000F000Fu>(w, 4);
        const uint32_t a2 = code_pair<0x000F000Fu>(w, 8), a3 = code_pair<0x000F000Fu>(w, 12);
        uint32_t h0 = 0, h1 = 0, h2 = 0, h3 = 0;
        if (BITS == 8) {
            const uint32_t hw = lds32(qp + kLoBytes + r * 128 + 4 * lane);
            h0 = code_pair<0x000F000Fu>(hw, 0);
            h1 = code_pair<0x000F000Fu>(hw, 4);
            h2 = code_pair<0x000F000Fu>(hw, 8);
            h3 = code_pair<0x000F000Fu>(hw, 12);
        }
        if (BITS == 6) {
            const uint32_t hw = __byte_perm(lds16(qp + kLoBytes + r * 64 + 2 * lane), 0u, 0x4140);
            h0 = code_pair<0x00030003u>(hw, 0);
            h1 = code_pair<0x00030003u>(hw, 2);
            h2 = code_pair<0x00030003u>(hw, 4);
            h3 = code_pair<0x00030003u>(hw, 6);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int i = 0; i < 4; ++i) c[r][nt][i] = d[r][nt][i] = 0.f;
            // one token: h hi and lo into one accumulator (fewer live registers; the four row
            // blocks still run in parallel)
            float (&dd)[4] = ONE ? c[r][nt] : d[r][nt];
            mma16816(c[r][nt], a0, a1, a2, a3, dc.hb[nt][0], dc.hb[nt][1]);
            mma16816(dd, a0, a1, a2, a3, dc.lb[nt][0], dc.lb[nt][1]);
            if (BITS != 4) {
                mma16816(c[r][nt], h0, h1, h2, h3, dc.hb16[nt][0], dc.hb16[nt][1]);
                mma16816(dd, h0, h1, h2, h3, dc.lb16[nt][0], dc.lb16[nt][1]);
            }
        }
    }
    const float off = (BITS == 4) ? 128.f : 2176.f;   // 128 per plane, the hi plane weighted 16x
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const uint2 sz = lds64(szp + r * 64 + 8 * g);
        const float sA = half_lo(sz.x), zA = half_hi(sz.x), sB = half_lo(sz.y), zB = half_hi(sz.y);
        const float oA = off + zA, oB = off + zB;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            acc[r][nt][0] += (sA * dc.w0[nt]) * ((c[r][nt][0] + d[r][nt][0]) - oA * dc.X0[nt]);
            acc[r][nt][2] += (sB * dc.w0[nt]) * ((c[r][nt][2] + d[r][nt][2]) - oB * dc.X0[nt]);
            if (!ONE) {
                acc[r][nt][1] += (sA * dc.w1[nt]) * ((c[r][nt][1] + d[r][nt][1]) - oA * dc.X1[nt]);
                acc[r][nt][3] += (sB * dc.w1[nt]) * ((c[r][nt][3] + d[r][nt][3]) - oB * dc.X1[nt]);
            }
        }
    }
}

// Adds one super-tile's accumulators into the fp32 output: rows 64 st + 16 r + g (+8), the
// tokens of the lane's columns (pairs pf + nt * 8 + 2t + col of the slot, nj of them).
template <int NT>
__device__ __forceinline__ void emit_st(const DecodeArgs &a, const DecodeSmem &S, int pf, int nj, int st,
                                        const float (&acc)[4][NT][4], int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int col = 0; col < 2; ++col) {
            const int q = nt * 8 + 2 * t + col;
            if (q < nj) {
                float *o = a.out_acc + (size_t)S.ptok[pf + q] * a.H + 64 * st + g;
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    red_add_f32(o + 16 * r, acc[r][nt][col]);
                    red_add_f32(o + 16 * r + 8, acc[r][nt][2 + col]);
                }
            }
        }
}

// ------------------------------------------------------------------------------ kernel
// NT: MMA n-tiles (8 tokens each) per unit; CW: consumer warps; STW: how a warp keeps the output
// rows of its super-tiles across units: > 0, in registers, STW super-tiles per warp (several
// tokens: the units of one expert slot); 0, not at all (each super-tile's rows are added out at
// once); -1, in shared memory (one token: all units of the CTA). NG: consumer groups; with two,
// group i (CW / 2 warps) runs the CTA's units i, i + 2, ... with its own barriers and h buffers,
// so that one group's barriers and SiLU-GLU overlap the other group's multiplications.
template <int NT, int STW, int CW, int NG>
__global__ void __launch_bounds__((CW + 1) * 32, 1) decode_kernel(const __grid_constant__ DecodeArgs a, const DecodeLayout L) {
    constexpr int kCW = CW, kPW = CW, kWarps = CW + 1, kThreads = kWarps * 32;
    constexpr int GW = CW / NG;   // warps per consumer group
    static_assert(NG == 1 || (NG == 2 && STW <= 0), "two groups: no register carry of output rows");
    extern __shared__ __align__(128) uint8_t dyn[];
    DecodeSmem &S = *reinterpret_cast<DecodeSmem *>(dyn);
    uint8_t *ring = dyn + L.ring;
    float *Xs = reinterpret_cast<float *>(dyn + L.xsum);
    float *gred = reinterpret_cast<float *>(dyn + L.gred);
    float *ycta_all = reinterpret_cast<float *>(dyn + L.ycta);
    const int NS = L.stages;
    const int T = a.T, H = a.H, E = a.E, K = a.k, P = T * K;
    const int G = H / kGroup, nst = H / 64;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nC = gridDim.x, c = blockIdx.x;
    uint32_t *status = &a.ctl->status;
    const bool xs_on = (size_t)T * H * 2 <= (size_t)kActBytes;
    const uint16_t *xsm = reinterpret_cast<const uint16_t *>(dyn + L.xs);
    const int ne = (E > c) ? (E - c + nC - 1) / nC : 0;   // router rows of this CTA: c, c+nC, ...
    const bool wr_on = (size_t)ne * H * 4 <= (size_t)NS * kStageBytes;
    const float *wsm = reinterpret_cast<const float *>(ring);
    const uint64_t drain_ns = a.wait_ns > 1000000ull ? a.wait_ns : 1000000ull;

    // ---------------------------------------------------------------- prologue (weights only)
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(&S.full[s]), 1);
            mbar_init(smem_u32(&S.empty[s]), kCW);
        }
        mbar_init(smem_u32(&S.wbar), 1);
        mbar_init(smem_u32(&S.xbar), 1);
        fence_barrier_init();
        S.abort = 0;
        if (wr_on && ne > 0) {
            const uint32_t rowb = (uint32_t)H * 4;
            mbar_expect_tx(smem_u32(&S.wbar), rowb * ne);
            for (int i = 0; i < ne; ++i)
                bulk_g2s(smem_u32(ring + (size_t)i * rowb), a.wr + (size_t)(c + i * nC) * H, rowb, smem_u32(&S.wbar));
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
    if (threadIdx.x < 3) S.wplan[threadIdx.x] = make_width_plan(H, a.I, 4 + 2 * threadIdx.x);
    if (STW < 0)
        for (int i = threadIdx.x; i < NG * H; i += kThreads) ycta_all[i] = 0.f;
    // the router bias of this CTA's rows (a weight), off the logits' critical path
    if (threadIdx.x < ne && threadIdx.x < kBiasRows) S.bias[threadIdx.x] = a.bias ? a.bias[c + threadIdx.x * nC] : 0.f;
    __syncthreads();
    // Everything below may read data that the previous launch in the stream produces.
    grid_dep_wait();

    // ---------------------------------------------------------------- logits
    if (threadIdx.x == 0) {
        // the copy of x first: the read of the call counter overlaps it
        if (xs_on) {
            const uint32_t bytes = (uint32_t)(T * H * 2);
            mbar_expect_tx(smem_u32(&S.xbar), bytes);
            bulk_g2s(smem_u32(dyn + L.xs), a.x, bytes, smem_u32(&S.xbar));
        }
        S.epoch = *reinterpret_cast<volatile unsigned long long *>(&a.ctl->done) / (unsigned long long)nC;
    }
    if (xs_on && !mbar_wait_idle(smem_u32(&S.xbar), 0, a.wait_ns, status)) S.abort = 1;
    if (wr_on && ne > 0 && !mbar_wait_idle(smem_u32(&S.wbar), 0, a.wait_ns, status)) S.abort = 1;
    __syncthreads();
    const unsigned long long epoch = S.epoch;
    const uint32_t tag = (uint32_t)(epoch + 1ull);
    const uint16_t *xr = xs_on ? xsm : a.x;
    // The CTA's ne * T dot products over H. With fewer of them than warps each is split into
    // slices of whole 256-element strides, one slice per warp, and the slices' sums are added
    // in slice order. Every logit word goes to lrep copies of the T x E block (lstride words
    // apart, spread over the L2 slices); CTA c polls copy c mod lrep.
    auto row_bias = [&](int i, int e) -> float { return i < kBiasRows ? S.bias[i] : (a.bias ? a.bias[e] : 0.f); };
    // every lane r < lrep stores copy r of a logit word
    auto publish_logit = [&](int t, int e, float l) {
        const unsigned long long w = ((unsigned long long)tag << 32) | (unsigned long long)__float_as_uint(l);
        if (lane < a.lrep) st_relaxed_u64(a.logits + (size_t)lane * a.lstride + (size_t)t * E + e, w);
    };
    // slices: nsl = 2^lsh per dot product, each lsl elements (a multiple of 256), so that the
    // CTA's dot products spread over its warps without integer division
    const int nq = ne * T, nsl = 1 << a.lsh;
    for (int it = warp; it < nq * nsl; it += kWarps) {
        const int q = it >> a.lsh, sl = it & (nsl - 1);
        const int i = T == 1 ? q : q / T, t = T == 1 ? 0 : q - (q / T) * T;
        const int e = c + i * nC;
        const float *wrow = wr_on ? wsm + (size_t)i * H : a.wr + (size_t)e * H;
        const uint16_t *xrow = xr + (size_t)t * H;
        const int h1 = min(H, (sl + 1) * a.lsl);
        float acc0 = 0.f, acc1 = 0.f;
        for (int h = sl * a.lsl + lane * 8; h < h1; h += 256) {
            const float4 w0 = *reinterpret_cast<const float4 *>(wrow + h);
            const float4 w1 = *reinterpret_cast<const float4 *>(wrow + h + 4);
            const uint4 xv = xs_on ? *reinterpret_cast<const uint4 *>(xrow + h) : __ldcg(reinterpret_cast<const uint4 *>(xrow + h));
            acc0 += w0.x * __uint_as_float(xv.x << 16) + w0.y * __uint_as_float(xv.x & 0xFFFF0000u);
            acc1 += w0.z * __uint_as_float(xv.y << 16) + w0.w * __uint_as_float(xv.y & 0xFFFF0000u);
            acc0 += w1.x * __uint_as_float(xv.z << 16) + w1.y * __uint_as_float(xv.z & 0xFFFF0000u);
            acc1 += w1.z * __uint_as_float(xv.w << 16) + w1.w * __uint_as_float(xv.w & 0xFFFF0000u);
        }
        float acc = acc0 + acc1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (nsl == 1) publish_logit(t, e, acc + row_bias(i, e));
        else if (lane == 0) S.lpart[it] = acc;
    }
    if (nsl > 1) {
        // the slices' sums added in slice order (the same logit bits on every run)
        __syncthreads();
        for (int q = warp; q < nq; q += kWarps) {
            const int i = T == 1 ? q : q / T, t = T == 1 ? 0 : q - (q / T) * T;
            const int e = c + i * nC;
            float l = 0.f;
            for (int sl = 0; sl < nsl; ++sl) l += S.lpart[q * nsl + sl];
            publish_logit(t, e, l + row_bias(i, e));
        }
    }
    grid_dep_launch();

    // per-token sums of x over each group, eight threads per group; with one token they are
    // formed by the consumer warps while the control warp routes
    auto group_sums = [&](int tid0, int nthreads) {
        const int n = T * G * 8;
        for (int base = tid0 - lane; base < n; base += nthreads) {
            const int i = base + lane;
            float s = 0.f;
            if (i < n) {
                const uint16_t *src = xr + (size_t)(i >> 3) * kGroup + (i & 7) * 8;
                const uint4 v = xs_on ? *reinterpret_cast<const uint4 *>(src) : __ldcg(reinterpret_cast<const uint4 *>(src));
                s = (__uint_as_float(v.x << 16) + __uint_as_float(v.x & 0xFFFF0000u)) +
                    (__uint_as_float(v.y << 16) + __uint_as_float(v.y & 0xFFFF0000u)) +
                    (__uint_as_float(v.z << 16) + __uint_as_float(v.z & 0xFFFF0000u)) +
                    (__uint_as_float(v.w << 16) + __uint_as_float(v.w & 0xFFFF0000u));
            }
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            s += __shfl_xor_sync(0xffffffffu, s, 4);
            if (i < n && (i & 7) == 0) Xs[i >> 3] = s;
        }
    };
    // ---------------------------------------------------------------- top-k (every CTA) + plan
    auto route_token = [&](int t) {
        const bool ok = !S.abort && (E <= 256 ? (K <= 8 ? token_topk_merge(a, S, t, tag, lane, c) : token_topk(a, S, t, tag, lane, c))
                                              : token_topk_wide(a, S, t, tag, lane, c));
        if (!ok && lane == 0) S.abort = 1;
    };
    const bool one = T == 1 && E <= 32 * kWarps;   // one token: the whole CTA routes it
    if (one) {
        const int nw = (E + 31) >> 5;
        if (warp < nw && !S.abort && !topk_one_candidates(a, S, tag, warp, lane) && lane == 0) S.abort = 1;
        __syncthreads();
        if (!S.abort) topk_one_rank(a, S, nw);
        __syncthreads();
        if (warp != kPW) group_sums(threadIdx.x, kCW * 32);
    } else {
        // tokens go to warps from the control warp on, so that with one token the control warp
        // routes it and makes the plan without a CTA barrier in between
        for (int t = (warp + 1) % kWarps; t < T; t += kWarps) route_token(t);
        if (warp != kPW || T > 1) group_sums(threadIdx.x, T > 1 ? kThreads : kCW * 32);
        if (T > 1) __syncthreads();
    }
    if (warp == kPW) {
        __syncwarp();
        // one token: the slots and the unit cut from the ranked selection, the first copies, and
        // only then the softmax weights (the consumers need them for the down step, the copies
        // do not)
        const bool sel_ok = !S.abort;
        if (one && sel_ok) topk_one_select(a, S, lane);
        const int Pp = sel_ok ? P : 0;
        if (T == 1) plan_single(S, Pp, lane, !one);
        else plan_many(a, S, Pp, lane);
        plan_units(a, S, lane, c, nC);
        // ------------------------------------------------------------ producer
        // The copies of chunk cc (in unit order) go to stage cc % NS. The first NS chunks find
        // every stage free: lane cc issues chunk cc, all at once; lane 0 then issues the rest,
        // each after its stage is released.
        uint32_t cc = 0;
        bool ok = true;
        const int sp = a.I / kSlice;
        auto walk = [&](bool fill) {
            int s = 0;
            uint32_t use = 0;
            int j = S.u0 / sp, i = S.u0 - (S.u0 / sp) * sp;   // slot and slice of the current unit
            for (int u = S.u0; u < S.u1 && ok; ++u) {
                const WidthPlan w = S.wplan[width_index(S.ubits[j])];
                const UnitGeo ug = unit_geo(a, S, w, j, i);
                for (int ch = 0; ch < w.ngc + w.ndc; ++ch) {
                    if (fill ? (use > 0) : false) return;
                    const bool mine = fill ? (int)cc == lane : use > 0;
                    if (!fill && use > 0 &&
                        (S.abort || !mbar_wait_idle(smem_u32(&S.empty[s]), (use - 1) & 1u, a.wait_ns, status))) {
                        S.abort = 1;
                        ok = false;
                        return;
                    }
                    if (mine) {
                        const uint32_t fb = smem_u32(&S.full[s]);
                        const uint32_t dst = smem_u32(ring + (size_t)s * kStageBytes);
                        int b0, b1;
                        if (ch < w.ngc) {
                            chunk_items(w.gbase, w.grem, ch, b0, b1);
                            const uint32_t bytes = (uint32_t)((b1 - b0) * 2 * w.tb);
                            mbar_expect_tx(fb, bytes);
                            bulk_g2s(dst, ug.gu + (size_t)b0 * 2 * w.tb, bytes, fb);
                        } else {
                            chunk_items(w.dbase, w.drem, ch - w.ngc, b0, b1);
                            const uint32_t zb = (uint32_t)((b1 - b0) * 256), qbytes = (uint32_t)((b1 - b0) * w.qb);
                            mbar_expect_tx(fb, zb + qbytes);
                            bulk_g2s(dst, ug.sz + (size_t)b0 * 256, zb, fb);
                            bulk_g2s(dst + zb, ug.q + (size_t)b0 * w.qb, qbytes, fb);
                        }
                    }
                    ++cc;
                    if (++s == NS) {
                        s = 0;
                        ++use;
                    }
                }
                if (++i == sp) {
                    i = 0;
                    ++j;
                }
            }
        };
        walk(true);
        __syncwarp();
        if (one && sel_ok) topk_one_finish(a, S, lane, c);
        // hand the plan to the consumer warps and stream the rest without waiting for them
        plan_ready_arrive<CW>();
        if (lane != 0) return;
        cc = 0;
        walk(false);
        // copies still in flight land before the CTA may exit (bounded by at least 1 ms, also when
        // the wait limit is 0)
        for (uint32_t q = cc > (uint32_t)NS ? cc - NS : 0; q < cc; ++q)
            mbar_wait(smem_u32(&S.full[q % NS]), (q / NS) & 1u, drain_ns, status);
        return;
    }

    // ---------------------------------------------------------------- consumers
    plan_ready_wait<CW>();
    const int g = lane >> 2, t = lane & 3;
    const int cg = NG == 1 ? 0 : warp / GW;    // this warp's consumer group
    const int gw = warp - cg * GW;             // and its warp within the group
    uint16_t *hhi = reinterpret_cast<uint16_t *>(dyn + L.hbuf) + (size_t)cg * 2 * NT * 8 * 16;
    uint16_t *hlo = hhi + NT * 8 * 16;
    float *hrow = reinterpret_cast<float *>(dyn + L.hcol) + (size_t)cg * 16 * NT * 8;
    float *ycta = ycta_all + (size_t)cg * H;
    // one token (STW = -1): only accumulator column 0 holds a pair, and the output rows are added
    // into shared memory
    constexpr bool ONE = STW < 0;
    constexpr int NL = STW > 0 ? STW : 1;
    static_assert(!ONE || NT == 1, "one token takes one n-tile");
    float yacc[NL][4][NT][4];
    auto zero_y = [&]() {
#pragma unroll
        for (int l = 0; l < NL; ++l)
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) yacc[l][r][nt][0] = yacc[l][r][nt][1] = yacc[l][r][nt][2] = yacc[l][r][nt][3] = 0.f;
    };
    zero_y();
    GuCtx<NT> jc;
    jc.bg = !xs_on;
    int s = 0;
    uint32_t par = 0;
    bool bad = false, aborted = false;
    int cur = -1, cur_pf = 0, cur_nj = 0;
    // the carried output rows of the current slot (several tokens: its pairs' tokens)
    auto flush_slot = [&]() {
        if (STW > 0) {
#pragma unroll
            for (int l = 0; l < NL; ++l) {
                const int st = warp + l * kCW;
                if (st < nst) emit_st<NT>(a, S, cur_pf, cur_nj, st, yacc[l], lane);
            }
            zero_y();
        }
    };
    auto next_stage = [&]() {
        if (++s == NS) {
            s = 0;
            par ^= 1u;
        }
    };
    // the lanes leave the bounded poll at different iterations: the vote makes the outcome
    // warp-uniform and reconverges the warp before its next aligned instruction (mma.sync, bar)
    auto wait_full = [&]() {
        if (!bad && (S.abort || !mbar_wait_idle(smem_u32(&S.full[s]), par, a.wait_ns, status))) bad = true;
        bad = __any_sync(0xffffffffu, bad);
    };
    auto release_stage = [&]() {
        __syncwarp();
        if (!bad && lane == 0) mbar_arrive(smem_u32(&S.empty[s]));
        next_stage();
    };
    const int sp = a.I / kSlice;
    int uj = S.u0 / sp, ui = S.u0 - (S.u0 / sp) * sp;   // slot and slice of the current unit
    for (int u = S.u0; u < S.u1; ++u) {
        const int bits = S.ubits[uj];
        const WidthPlan w = S.wplan[width_index(bits)];
        if (NG > 1 && ((u - S.u0) & (NG - 1)) != cg) {
            // the other group's unit: every consumer warp still waits for each chunk and releases
            // it (without reading it), so that both groups pass the ring's stages in order: a
            // stage's phase parity only tells consecutive phases apart, and a group more than one
            // phase ahead of or behind a stage would misread it
            for (int ch = 0; ch < w.ngc + w.ndc; ++ch) {
                wait_full();
                release_stage();
            }
            if (++ui == sp) {
                ui = 0;
                ++uj;
            }
            continue;
        }
        if (uj != cur) {
            if (T > 1 && cur >= 0 && !bad) flush_slot();
            cur = uj;
            cur_pf = S.pfirst[cur];
            cur_nj = S.pfirst[cur + 1] - cur_pf;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int q = nt * 8 + g, q0 = nt * 8 + 2 * t, q1 = q0 + 1;
                const int tok = S.ptok[cur_pf + (q < cur_nj ? q : 0)];
                jc.b[nt] = a.x + (size_t)tok * H;
                jc.sb[nt] = smem_u32(xsm) + (uint32_t)(tok * H * 2);
                jc.xs0[nt] = smem_u32(Xs) + (uint32_t)(S.ptok[cur_pf + (q0 < cur_nj ? q0 : 0)] * G * 4);
                jc.xs1[nt] = smem_u32(Xs) + (uint32_t)(S.ptok[cur_pf + (q1 < cur_nj ? q1 : 0)] * G * 4);
            }
        }
        if (++ui == sp) {
            ui = 0;
            ++uj;
        }
        const int ngc = w.ngc, ndc = w.ndc, qb = w.qb;
        // gate/up: split K over the warps, partial sums into shared memory
        float gacc[2][NT][4];
#pragma unroll
        for (int rb = 0; rb < 2; ++rb)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) gacc[rb][nt][0] = gacc[rb][nt][1] = gacc[rb][nt][2] = gacc[rb][nt][3] = 0.f;
        for (int ch = 0; ch < ngc; ++ch) {
            wait_full();
            if (!bad) {
                int k0, k1;
                chunk_items(w.gbase, w.grem, ch, k0, k1);
                const uint8_t *stg = ring + (size_t)s * kStageBytes;
                if (bits == 4) gu_chunk<4, NT, GW, ONE>(stg, k0, k1, gw, jc, lane, gacc);
                else if (bits == 6) gu_chunk<6, NT, GW, ONE>(stg, k0, k1, gw, jc, lane, gacc);
                else gu_chunk<8, NT, GW, ONE>(stg, k0, k1, gw, jc, lane, gacc);
            }
            release_stage();
        }
        // each warp's partial sums into its own slice of shared memory (plain stores)
        if (!bad) {
            float *gw = gred + (size_t)warp * 2 * NT * 4 * 32 + lane;
#pragma unroll
            for (int rb = 0; rb < 2; ++rb)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) gw[((rb * NT + nt) * 4 + i) * 32] = gacc[rb][nt][i];
        }
        if (group_sync_or<NG, CW>(cg, bad || S.abort)) {
            aborted = true;
            break;
        }
        // SiLU-GLU, one intermediate row k of the unit per warp of the group (warps k, k + GW),
        // one pair column per lane: the gate and up sums over the group's partials, h as a bf16
        // hi + lo pair, and hi + lo of every (row, column) for the down step's correction sums.
        for (int k = gw; k < 16; k += GW) {
            if (lane < 8 * NT) {
                const int nt = lane >> 3, pcol = lane & 7;
                const int rb = k >> 3, src = ((k & 7) << 2) + (pcol >> 1), col = pcol & 1;
                const float *gp = gred + (size_t)cg * GW * 2 * NT * 4 * 32 + ((rb * NT + nt) * 4 + col) * 32 + src;
                // the warps' partials, summed as a tree (all loads first)
                float gv[GW], uv[GW];
#pragma unroll
                for (int w2 = 0; w2 < GW; ++w2) {
                    gv[w2] = gp[(size_t)w2 * 2 * NT * 4 * 32];
                    uv[w2] = gp[(size_t)w2 * 2 * NT * 4 * 32 + 2 * 32];
                }
#pragma unroll
                for (int h = GW / 2; h > 0; h >>= 1)
#pragma unroll
                    for (int w2 = 0; w2 < h; ++w2) {
                        gv[w2] += gv[w2 + h];
                        uv[w2] += uv[w2 + h];
                    }
                const float gt = gv[0], up = uv[0];
                const float h = __fdividef(gt, 1.f + __expf(-gt)) * up;
                const __nv_bfloat16 hi = __float2bfloat16_rn(h);
                const __nv_bfloat16 lo = __float2bfloat16_rn(h - __bfloat162float(hi));
                const int o = (nt * 8 + pcol) * 16 + k;
                hhi[o] = __bfloat16_as_ushort(hi);
                hlo[o] = __bfloat16_as_ushort(lo);
                hrow[k * NT * 8 + lane] = __bfloat162float(hi) + __bfloat162float(lo);
            }
        }
        group_sync<NG, CW>(cg);
        DnCtx<NT> dc;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint32_t o = (uint32_t)(((nt * 8 + g) * 16 + 4 * t) * 2);
            const uint2 vh = lds64(smem_u32(hhi) + o), vl = lds64(smem_u32(hlo) + o);
            dc.hb[nt][0] = vh.x;
            dc.hb[nt][1] = vh.y;
            dc.lb[nt][0] = vl.x;
            dc.lb[nt][1] = vl.y;
            if (bits != 4) {
                dc.hb16[nt][0] = bf16x2_mul16(vh.x);
                dc.hb16[nt][1] = bf16x2_mul16(vh.y);
                dc.lb16[nt][0] = bf16x2_mul16(vl.x);
                dc.lb16[nt][1] = bf16x2_mul16(vl.y);
            } else {
                dc.hb16[nt][0] = dc.hb16[nt][1] = dc.lb16[nt][0] = dc.lb16[nt][1] = 0u;
            }
            // X of the lane's accumulator columns (pairs 2t, 2t + 1): the sums over the 16 rows
            float xa[16], xb[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float2 v = *reinterpret_cast<const float2 *>(hrow + k * NT * 8 + nt * 8 + 2 * t);
                xa[k] = v.x;
                xb[k] = v.y;
            }
#pragma unroll
            for (int h = 8; h > 0; h >>= 1)
#pragma unroll
                for (int k = 0; k < h; ++k) {
                    xa[k] += xa[k + h];
                    xb[k] += xb[k + h];
                }
            const float x0 = xa[0], x1 = xb[0];
            dc.X0[nt] = x0;
            dc.X1[nt] = x1;
            const int q0 = nt * 8 + 2 * t, q1 = q0 + 1;
            dc.w0[nt] = q0 < cur_nj ? S.pw[cur_pf + q0] : 0.f;
            dc.w1[nt] = q1 < cur_nj ? S.pw[cur_pf + q1] : 0.f;
        }
        // down: super-tile st of the unit's quarter goes to warp st % GW of the group
        for (int ch = 0; ch < ndc; ++ch) {
            wait_full();
            if (!bad) {
                int s0, s1;
                chunk_items(w.dbase, w.drem, ch, s0, s1);
                const uint32_t zb = smem_u32(ring + (size_t)s * kStageBytes), qbase = zb + (uint32_t)((s1 - s0) * 256);
                if (STW > 0) {
#pragma unroll
                    for (int l = 0; l < NL; ++l) {
                        const int st = warp + l * kCW;
                        if (st >= s0 && st < s1) {
                            const uint32_t zp = zb + (uint32_t)((st - s0) * 256), qp = qbase + (uint32_t)((st - s0) * qb);
                            if (bits == 4) down_st<4, NT, ONE>(zp, qp, dc, lane, yacc[l]);
                            else if (bits == 6) down_st<6, NT, ONE>(zp, qp, dc, lane, yacc[l]);
                            else down_st<8, NT, ONE>(zp, qp, dc, lane, yacc[l]);
                        }
                    }
                } else {
                    for (int st = s0 + ((gw - s0) % GW + GW) % GW; st < s1; st += GW) {
                        const uint32_t zp = zb + (uint32_t)((st - s0) * 256), qp = qbase + (uint32_t)((st - s0) * qb);
                        if (bits == 4) down_st<4, NT, ONE>(zp, qp, dc, lane, yacc[0]);
                        else if (bits == 6) down_st<6, NT, ONE>(zp, qp, dc, lane, yacc[0]);
                        else down_st<8, NT, ONE>(zp, qp, dc, lane, yacc[0]);
                        if (STW == 0) {
                            emit_st<NT>(a, S, cur_pf, cur_nj, st, yacc[0], lane);
                        } else if (t == 0) {
                            // one token (column 0): this warp owns the super-tile's rows
#pragma unroll
                            for (int r = 0; r < 4; ++r) {
                                ycta[64 * st + 16 * r + g] += yacc[0][r][0][0];
                                ycta[64 * st + 16 * r + g + 8] += yacc[0][r][0][2];
                            }
                        }
                        zero_y();
                    }
                }
            }
            release_stage();
        }
    }
    if (!aborted && consumer_sync_or<CW>(bad || S.abort)) aborted = true;
    // ---------------------------------------------------------------- output rows
    if (!aborted && S.u1 > S.u0) {
        if (STW < 0) {
            // one token: the CTA's rows, one vector addition per 4 rows
            consumer_sync<CW>();
            for (int i = threadIdx.x; i < H / 4; i += kCW * 32) {
                float4 v = reinterpret_cast<const float4 *>(ycta_all)[i];
                if (NG > 1) {
                    const float4 v2 = reinterpret_cast<const float4 *>(ycta_all + H)[i];
                    v.x += v2.x;
                    v.y += v2.y;
                    v.z += v2.z;
                    v.w += v2.w;
                }
                red_add_v4_f32(a.out_acc + 4 * i, v);
            }
        } else if (STW > 0) {
            flush_slot();
        }
    }
    // ---------------------------------------------------------------- completion
    // Each row group's counter grows by one per CTA and call; the CTA whose addition completes a
    // call's count converts the group to bf16 and clears it (release of this CTA's additions,
    // ordered before by the barrier, and acquire of the others', in one step).
    consumer_sync<CW>();
    const int ngr = (H + kRowGroup - 1) / kRowGroup;
    for (int gi = warp; gi < ngr; gi += kCW) {
        int last = 0;
        if (lane == 0) {
            const unsigned long long old = atom_add_acq_rel_u64(a.rowcnt + gi, 1ull);
            last = ((old + 1ull) % (unsigned long long)nC) == 0ull ? 1 : 0;
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        __syncwarp();
        if (last) {
            const int r0 = gi * kRowGroup, n4 = (min(H, r0 + kRowGroup) - r0) / 4;
            for (int i = lane; i < T * n4; i += 32) {
                const int tt = i / n4, c4 = i - tt * n4;
                float4 *p = reinterpret_cast<float4 *>(a.out_acc + (size_t)tt * H + r0) + c4;
                const float4 v = __ldcg(p);
                const __nv_bfloat162 lo2 = __floats2bfloat162_rn(v.x, v.y), hi2 = __floats2bfloat162_rn(v.z, v.w);
                reinterpret_cast<uint2 *>(a.out + (size_t)tt * H + r0)[c4] =
                    make_uint2(*reinterpret_cast<const uint32_t *>(&lo2), *reinterpret_cast<const uint32_t *>(&hi2));
                __stcg(p, make_float4(0.f, 0.f, 0.f, 0.f));
            }
        }
    }
    if (threadIdx.x == 0) {
        atomicAdd(&a.ctl->done, 1ull);
        // the prologue's copies have landed before the CTA exits (they may not have if a wait
        // for them expired)
        if (xs_on) mbar_wait(smem_u32(&S.xbar), 0, drain_ns, status);
        if (wr_on && ne > 0) mbar_wait(smem_u32(&S.wbar), 0, drain_ns, status);
    }
}

// Copies of the exchanged logit words within the fixed logit region (kMaxT x kMaxE words): the
// T x E block at 4 KB-aligned strides, up to 32 copies.
void logit_copies(int T, int E, int &rep, int &stride) {
    stride = (int)align_up((size_t)T * E, 512);
    rep = 1;
    while (rep < 32 && (size_t)(rep * 2) * stride <= (size_t)kMaxT * kMaxE) rep *= 2;
}

template <int NT, int STW, int CW, int NG>
moe_status_t launch_nt(const DecodeArgs &a, const DeviceInfo *dev, cudaStream_t st) {
    const DecodeLayout L = decode_layout<NT, CW, NG>(a.T, a.H, dev->max_smem_optin);
    if (L.stages < 2) return MOE_ERR_UNSUPPORTED;
    // the kernel attribute, once per device (concurrent first calls from several host threads
    // set the same value; the flag is atomic)
    static std::atomic<bool> attr_set[64];
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64) return MOE_ERR_CUDA;
    if (!attr_set[d].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(decode_kernel<NT, STW, CW, NG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dev->max_smem_optin) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_set[d].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(dev->sms);
    cfg.blockDim = dim3((CW + 1) * 32);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, decode_kernel<NT, STW, CW, NG>, a, L) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

}  // namespace

moe_status_t launch_decode(const uint16_t *x, const float *wr, const float *bias, const void *packed,
                           int T, int H, int I, int E, int k, uint16_t *out, int32_t *idx_out,
                           float *w_out, void *ws, cudaStream_t st) {
    if (T * k > kMaxP || T > kMaxT || H > kDecodeMaxH) return MOE_ERR_UNSUPPORTED;
    const DeviceInfo *dev = device_info();
    if (!dev) return MOE_ERR_CUDA;
    const DecodeWs W = decode_ws_layout(T, H, I, E, k);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    DecodeArgs a;
    a.x = x; a.wr = wr; a.bias = bias; a.packed = static_cast<const uint8_t *>(packed);
    a.T = T; a.H = H; a.I = I; a.E = E; a.k = k;
    a.out = out; a.idx_out = idx_out; a.w_out = w_out;
    a.ctl = reinterpret_cast<Control *>(w8);
    a.logits = reinterpret_cast<unsigned long long *>(w8 + W.logits);
    a.rowcnt = reinterpret_cast<unsigned long long *>(w8 + W.rowcnt);
    a.out_acc = reinterpret_cast<float *>(w8 + W.out_acc);
    a.wait_ns = wait_limit_ns();
    a.kmul = (uint32_t)((65536 + k - 1) / k);
    logit_copies(T, E, a.lrep, a.lstride);
    {
        // the most slices (a power of two dividing H / 256) that give every warp of the CTA with
        // the most router rows one dot-product slice at most
        const int warps = T == 1 ? 17 : (T <= 16 ? 17 : 9);
        const int nq = ((E + dev->sms - 1) / dev->sms) * T;
        const int nstr = (H + 255) / 256;
        int sh = 0;
        while (nstr % (2 << sh) == 0 && nq * (2 << sh) <= warps && (2 << sh) <= 4 * kMaxWarps / max(nq, 1)) ++sh;
        a.lsh = sh;
        a.lsl = (nstr >> sh) * 256;
    }
    // One token: 16 consumer warps, the CTA's output rows in shared memory. Several tokens: every
    // super-tile's rows are added into the output at once.
    if (T == 1) return launch_nt<1, -1, 16, MOE_DECODE_GROUPS>(a, dev, st);
    if (T <= 8) return launch_nt<1, 0, 16, MOE_DECODE_GROUPS>(a, dev, st);
    if (T <= 16) return launch_nt<2, 0, 16, MOE_DECODE_GROUPS>(a, dev, st);
    return launch_nt<4, 0, 8, 1>(a, dev, st);
}

}  // namespace moe
