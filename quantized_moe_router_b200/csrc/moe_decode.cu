// moe_decode.cu -- the decode megakernel: one persistent launch per layer computes routing,
// gate/up, SiLU-GLU, down and the weighted combine of the MoE expert block for T <= 32 tokens.
//
// This is the "MoE megakernel" of the page "Raon-1-mini ... RTX 5070 Ti" (table row: one
// persistent kernel for each layer's expert block) with the "pipelined megakernel" row's
// overlap (the next expert's tiles are in flight while the current one is multiplied), laid
// out for sm_100a. One CTA per SM: 8 consumer warps and one control warp.
//   * Prologue, before the programmatic-dependent-launch wait (it overlaps the previous
//     layer): mbarrier set-up, this CTA's router rows copied into shared memory, the packed
//     layer's expert table read. Both are weights, never produced by the previous launch.
//   * Routing. x is copied into shared memory; each CTA computes the fp32 logits of its
//     E / nCTA experts (the dot products split over all warps) and publishes each as one 8-byte
//     word {logit, call tag} into up to 32 copies of the T x E block, so that the CTAs' polls
//     spread over the L2 slices. Every CTA polls its copy until all words carry this call's tag
//     (derived from a completion counter that grows by nCTA per call: no barrier, no reset) and
//     runs the same top-k + softmax: all CTAs agree on the selection without a second exchange.
//   * Plan (control warp). Unique experts in ascending id, their pair lists (ascending token)
//     and two job sequences: gate/up jobs (8 intermediate rows x all of H) and down jobs (16
//     output rows x all of I). Each CTA takes a contiguous range of each, cut so that every CTA
//     streams the same number of bytes as a few long contiguous regions.
//   * Streaming. The control warp streams the CTA's regions with bulk copies of up to 48 KB
//     (on B200 one SM completes roughly one bulk copy per 250 ns whatever its size, and every
//     chunk costs the consumers one barrier, so chunks are large) into a ring of 2-3 stages,
//     writing each chunk's job range into a descriptor next to it.
//   * Gate/up: tile kg of a job goes to consumer warp kg % 8 (split K), which multiplies it with
//     mma.sync on bf16 operands made from the codes by one LOP3 per register (exact integers
//     128 + q) and applies the group's scale and zero in fp32; after its last tile of a job a
//     warp adds its partial into the job's shared-memory slot. One consumer barrier per chunk
//     marks the previous chunk's jobs complete; each is finalised (SiLU-GLU, h as a bf16 hi/lo
//     pair) by one warp while the others run on. The CTA publishes its h rows once (counter adds
//     per expert after a fence); a down job waits only for the counter of its own expert.
//   * Down: a whole job in one warp (its few tiles in a row), w * y added into the fp32 output
//     accumulator.
//   * The last CTA to finish (completion counter) converts the accumulator to bf16 and clears
//     the accumulator and the counters for the next call.
// Every wait is bounded; on expiry the kernel records MOE_ERR_TIMEOUT in the workspace, the
// warps skip the remaining work in lock step, and the call still leaves the workspace clean.
// The kernel is instantiated for 1, 2 and 4 MMA n-tiles (up to 8, 16 and 32 tokens per expert).
#include "moe_internal.cuh"
#include "moe_topk.cuh"

namespace moe {
namespace {

constexpr int kCW = 8;                      // consumer warps
constexpr int kWarps = kCW + 1;             // + the control warp (routing plan, bulk copies)
constexpr int kThreads = kWarps * 32;
constexpr int kStageBytes = 49152;          // bytes per bulk copy / ring stage
constexpr int kMaxStages = 8;
constexpr int kActBytes = 65536;            // x (routing + gate/up), then h of one expert (down)
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
    uint16_t *h_hi, *h_lo;
    float *out_acc;
    uint32_t *h_ready;
    uint64_t wait_ns;
    double rnC;                  // 1 / number of CTAs
    uint32_t cm, cs1, cs2;       // division by the number of CTAs: multiplier and shifts
    uint32_t kmul;               // ceil(2^16 / k): p / k = (p * kmul) >> 16 for p < 2048
    int lrep;                    // copies of the logit words (a power of two)
    int lstride;                 // words between copies
};

// One ring stage's chunk, written by the producer before it starts the copy: jobs job0 ..
// job0 + njobs - 1 of one phase and one expert slot u; the first job from its tile k0, the last
// up to tile k1 (tpj tiles per job); job0's tile 0 lies base_off bytes from the stage start
// (negative when the chunk begins inside that job). flags: 1 gate/up phase, 2 the CTA's last chunk.
struct __align__(16) ChunkDesc {
    int job0, base_off;
    short njobs, k0, k1, tpj;
    unsigned short tb;
    unsigned char bits, flags;
    short u, pad;
};

struct __align__(16) DecodeSmem {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t xbar, wbar;
    unsigned long long epoch;
    volatile int abort;
    int U, g0, g1, d0, d1, nGU;
    int is_last;
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
    float sel_w[kMaxP];
    float lpart[kWarps];                // slice sums of the router dot products
    ChunkDesc desc[kMaxStages];         // the chunk of each ring stage
    float bias[kBiasRows];              // router bias of the CTA's rows c, c + nCTA, ...
    __align__(16) uint32_t plist[32];   // plan scratch: packed pair list
};

// accumulator slots of NT n-tiles: 16 rows x 8*NT columns fp32, laid out as the MMA fragments
template <int NT> constexpr int slots_for() { return NT == 4 ? 8 : 16; }
// A gate/up job's partial sums stay in its slot from the chunk that completes it until the next
// chunk's barrier; meanwhile that chunk adds into the slots of the jobs it touches. A chunk touching at
// most (slots - 1) / 2 jobs keeps the two sets apart, so a chunk holds at most that minus one
// jobs' worth of tiles.
template <int NT> constexpr int chunk_jobs() { return (slots_for<NT>() - 1) / 2 - 1; }
template <int NT> constexpr int slot_floats() { return NT * 128; }

struct DecodeLayout {
    size_t ring, act, accs, xs, total;
    int stages;
};
template <int NT>
DecodeLayout decode_layout(int T, int H, int smem_limit) {
    DecodeLayout L;
    size_t o = align_up(sizeof(DecodeSmem), 128);
    L.act = o;
    o += kActBytes;
    L.accs = o;
    o += (size_t)slots_for<NT>() * slot_floats<NT>() * 4;
    L.xs = o;
    o += align_up((size_t)T * (H / kGroup) * 4, 128);
    L.ring = align_up(o, 128);
    const long long room = (long long)min(smem_limit, kSmemBudget) - (long long)L.ring;
    L.stages = room > 0 ? (int)(room / kStageBytes) : 0;
    if (L.stages > kMaxStages) L.stages = kMaxStages;
    L.total = L.ring + (size_t)L.stages * kStageBytes;
    return L;
}

__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory"); }
// The same barrier, returning the OR of `flag` over the consumer threads: a decision that all
// consumer warps take identically (S.abort can change at any time, so reading it after a plain
// barrier could split the warps).
__device__ __forceinline__ bool consumer_sync_or(bool flag) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)flag), "n"(kCW * 32)
        : "memory");
    return r != 0;
}
// named barrier 2: the control warp arrives when the plan is in shared memory, the consumer
// warps wait for it (and for each other's group sums)
__device__ __forceinline__ void plan_ready_arrive() { asm volatile("bar.arrive 2, %0;" ::"n"(kThreads) : "memory"); }
__device__ __forceinline__ void plan_ready_wait() { asm volatile("bar.sync 2, %0;" ::"n"(kThreads) : "memory"); }
__device__ __forceinline__ unsigned long long atom_add_acq_rel_u64(unsigned long long *p, unsigned long long v) {
    unsigned long long old;
    asm volatile("atom.acq_rel.gpu.global.add.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
    return old;
}
__device__ __forceinline__ void red_shared_f32(float *p, float v) {
    asm volatile("red.relaxed.cta.shared::cta.add.f32 [%0], %1;" ::"r"(smem_u32(p)), "f"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
// bounded spin on a global word reaching `target` (one thread); false on expiry
__device__ __forceinline__ bool wait_counter(const uint32_t *p, uint32_t target, uint64_t limit_ns,
                                             uint32_t *status) {
    if (ld_acquire_u32(p) >= target) return true;
    const uint64_t t0 = global_timer();
    while (true) {
        __nanosleep(64);
        if (ld_acquire_u32(p) >= target) return true;
        if (global_timer() - t0 > limit_ns) {
            atomicOr(status, kStatusTimeout);
            return false;
        }
    }
}

// ------------------------------------------------------------------------------ job layout
// A run of consecutive jobs of one expert and one phase: contiguous in the packed layer.
struct Region {
    const uint8_t *src;
    int tiles, tb, bits, u, rb0, jg0, tpj;   // jg0: global index of the first job
};

__device__ __forceinline__ Region region_at(const DecodeSmem &S, const DecodeArgs &a, bool gu, int j) {
    Region r;
    const int G = a.H / kGroup, GI = a.I / kGroup;
    const int per = gu ? a.I / 8 : a.H / 16;    // jobs per expert
    const int end = gu ? S.g1 : S.d1;
    r.u = j / per;
    r.rb0 = j % per;
    r.jg0 = j;
    const int jend = min(end, (r.u + 1) * per);
    r.tpj = gu ? G : GI;
    r.tiles = (jend - j) * r.tpj;
    r.bits = S.ubits[r.u];
    r.tb = tile_bytes(r.bits);
    const uint8_t *base = a.packed + (size_t)S.uoff[r.u] * 256;
    r.src = gu ? base + (size_t)r.rb0 * G * r.tb : base + gu_tiles(a.H, a.I) * r.tb + (size_t)r.rb0 * GI * r.tb;
    return r;
}
// Chunks of a region: at most one stage and at most maxjobs jobs' worth of tiles (gate/up
// chunks, whose jobs keep partial sums in slots).
__device__ __forceinline__ int region_chunks(const Region &r, int maxjobs) {
    const int cap = min(kStageBytes / r.tb, maxjobs * r.tpj);
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
// Operand sources of the current job for this lane: per n-tile, the row that the lane's B
// column reads (x row for gate/up, h hi row for down; null where the column has no token),
// the h lo row (down), and the group-sum rows of its two accumulator columns.
template <int NT>
struct JobCtx {
    const uint16_t *b[NT];   // global rows (bg) or null
    const uint16_t *b2[NT];
    uint32_t sb[NT], sb2[NT];    // shared-memory rows (!bg)
    uint32_t xs0[NT], xs1[NT];   // shared-memory group-sum rows
    bool has[NT], has0[NT], has1[NT];
    bool bg;   // B rows are in global memory (read through L2) rather than shared memory
};

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
// predicated shared-memory store (no branch)
__device__ __forceinline__ void sts_if(bool p, int *addr, int v) {
    asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %0, 0;\n\t@q st.shared.u32 [%1], %2;\n\t}" ::"r"((int)p),
                 "r"(smem_u32(addr)), "r"(v)
                 : "memory");
}
__device__ __forceinline__ float lds32f(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
    return v;
}

template <int BITS, int NT, bool GU>
__device__ __forceinline__ void consume_tile(const uint8_t *tile, int kg, const JobCtx<NT> &jc, int lane,
                                             float (&acc)[NT][4]) {
    const int g = lane >> 2, t = lane & 3;
    const uint4 lo = *reinterpret_cast<const uint4 *>(tile + 16 * lane);
    uint4 hi8 = make_uint4(0, 0, 0, 0);
    uint2 hi6 = make_uint2(0, 0);
    if (BITS == 8) hi8 = *reinterpret_cast<const uint4 *>(tile + kLoBytes + 16 * lane);
    if (BITS == 6) hi6 = *reinterpret_cast<const uint2 *>(tile + kLoBytes + 8 * lane);
    const uint2 sz = *reinterpret_cast<const uint2 *>(tile + kLoBytes + hi_bytes(BITS) + 8 * g);
    const float sA = half_lo(sz.x), zA = half_hi(sz.x), sB = half_lo(sz.y), zB = half_hi(sz.y);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        // Up to two n-tiles every lane loads: a column without a token reads a valid row (the
        // first pair's) and produces accumulator columns that nothing reads, with no divergent
        // branch per tile. Four n-tiles keep the guard (their registers are tight).
        uint32_t b[8] = {0, 0, 0, 0, 0, 0, 0, 0}, b2[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (NT <= 2 || jc.has[nt]) {
            uint4 v0, v1, w0 = make_uint4(0, 0, 0, 0), w1 = make_uint4(0, 0, 0, 0);
            if (jc.bg) {
                const uint4 *p = reinterpret_cast<const uint4 *>(jc.b[nt] + kg * kGroup + 16 * t);
                v0 = __ldcg(p);
                v1 = __ldcg(p + 1);
                if (!GU) {
                    const uint4 *p2 = reinterpret_cast<const uint4 *>(jc.b2[nt] + kg * kGroup + 16 * t);
                    w0 = __ldcg(p2);
                    w1 = __ldcg(p2 + 1);
                }
            } else {
                const uint32_t o = (uint32_t)(kg * kGroup + 16 * t) * 2;
                v0 = lds128(jc.sb[nt] + o);
                v1 = lds128(jc.sb[nt] + o + 16);
                if (!GU) {
                    w0 = lds128(jc.sb2[nt] + o);
                    w1 = lds128(jc.sb2[nt] + o + 16);
                }
            }
            b[0] = v0.x; b[1] = v0.y; b[2] = v0.z; b[3] = v0.w;
            b[4] = v1.x; b[5] = v1.y; b[6] = v1.z; b[7] = v1.w;
            b2[0] = w0.x; b2[1] = w0.y; b2[2] = w0.z; b2[3] = w0.w;
            b2[4] = w1.x; b2[5] = w1.y; b2[6] = w1.z; b2[7] = w1.w;
        }
        const float X0 = (NT <= 2 || jc.has0[nt]) ? lds32f(jc.xs0[nt] + kg * 4) : 0.f;
        const float X1 = (NT <= 2 || jc.has1[nt]) ? lds32f(jc.xs1[nt] + kg * 4) : 0.f;
        tile_group_mma<BITS>(lo, hi8, hi6, b, GU ? nullptr : b2, sA, zA, sB, zB, X0, X1, acc[nt]);
    }
}

// All tiles [k0, k1) of a job owned by one warp, two at a time.
template <int BITS, int NT>
__device__ __forceinline__ void run_tiles_seq(const uint8_t *job_base, int tb, int k0, int k1, const JobCtx<NT> &jc,
                                              int lane, float (&acc)[NT][4], float (&acc2)[NT][4]) {
    int kg = k0;
    for (; kg + 1 < k1; kg += 2) {
        consume_tile<BITS, NT, false>(job_base + (size_t)kg * tb, kg, jc, lane, acc);
        consume_tile<BITS, NT, false>(job_base + (size_t)(kg + 1) * tb, kg + 1, jc, lane, acc2);
    }
    if (kg < k1) consume_tile<BITS, NT, false>(job_base + (size_t)kg * tb, kg, jc, lane, acc);   // odd tail
}

// The warp's tiles of job `jb` (region-local) inside a chunk: k-tiles kg in [k0, k1) with
// kg % kCW == warp, two at a time so that their MMA chains interleave.
template <int BITS, int NT, bool GU>
__device__ __forceinline__ void run_tiles(const uint8_t *job_base, int tb, int k0, int k1, int warp,
                                          const JobCtx<NT> &jc, int lane, float (&acc)[NT][4],
                                          float (&acc2)[NT][4]) {
    int kg = k0 + ((warp - k0) % kCW + kCW) % kCW;   // first tile >= k0 with kg % kCW == warp
    for (; kg + kCW < k1; kg += 2 * kCW) {
        consume_tile<BITS, NT, GU>(job_base + (size_t)kg * tb, kg, jc, lane, acc);
        consume_tile<BITS, NT, GU>(job_base + (size_t)(kg + kCW) * tb, kg + kCW, jc, lane, acc2);
    }
    if (kg < k1) consume_tile<BITS, NT, GU>(job_base + (size_t)kg * tb, kg, jc, lane, acc);   // odd tail
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

// floor(X * cc / nC) without an integer division. Below 2^32 the product is divided by the
// invariant-divisor method of Granlund and Montgomery (a multiply-high, an add and two shifts
// with constants set up on the host, exact for every 32-bit dividend); above, the quotient is
// taken through the double reciprocal of nC (X * cc < 2^53 is exact in double and the estimate
// is floor or floor - 1) and corrected once.
__device__ __forceinline__ uint32_t cut_units(const DecodeArgs &a, uint32_t X, int cc, int nC) {
    const unsigned long long n = (unsigned long long)X * (unsigned)cc;
    if (n < (1ull << 32)) {
        const uint32_t n32 = (uint32_t)n, t = __umulhi(a.cm, n32);
        return (t + ((n32 - t) >> a.cs1)) >> a.cs2;
    }
    unsigned long long q = (unsigned long long)((double)n * a.rnC);
    q += ((q + 1ull) * (unsigned)nC <= n) ? 1ull : 0ull;
    return (uint32_t)q;
}
// Smallest r with r * d >= n, for results below 2^16: the truncated float quotient (relative
// error below 2^-20, so within 0.07 of n / d) is floor(n / d) - 1, floor(n / d) or ceil(n / d),
// and two conditional increments reach ceil(n / d).
__device__ __forceinline__ uint32_t ceil_div_small(uint32_t n, uint32_t d) {
    uint32_t r = (uint32_t)__fdividef((float)n, (float)d);
    r += ((unsigned long long)r * d < n) ? 1u : 0u;
    r += ((unsigned long long)r * d < n) ? 1u : 0u;
    return r;
}
// First job (of a gate/up or down sequence) whose first unit is at or after q, found by the
// lanes of a warp of which some hold one expert slot each (U <= 32 slots, in any lane order):
// such a lane holds the slot's index, its first unit lo, its end hi and its units per job jb;
// `per` jobs per slot, `total` units in all. The slot holding q is the one with lo < q <= hi
// (slot 0 for q = 0). `start` receives the job's first unit (total past the last job).
__device__ __forceinline__ int job_at_unit_warp(uint32_t lo, uint32_t hi, uint32_t jb, int slot, bool slot_lane,
                                                int per, int U, uint32_t q, uint32_t total, uint32_t &start) {
    const bool holds = slot_lane && (q == 0 ? lo == 0 : (lo < q && q <= hi));
    const uint32_t m = __ballot_sync(0xffffffffu, holds);
    const uint32_t r = holds ? ceil_div_small(q - lo, jb) : 0u;
    const uint32_t st = lo + r * jb;
    const int j = slot * per + (int)r;
    if (m == 0) {
        start = total;
        return U * per;
    }
    const int u = __ffs(m) - 1;
    start = __shfl_sync(0xffffffffu, st, u);
    return __shfl_sync(0xffffffffu, j, u);
}

__device__ __forceinline__ int slot_of(const DecodeSmem &S, int e) {
    const int w = e >> 5;
    return S.wordpre[w] + __popc(S.selmask[w] & ((1u << (e & 31)) - 1u));
}

// Plan for more than 32 pairs (several tokens), out of line: bitmap of the selection in shared
// memory, per-slot counts and a stable fill of the pair lists 32 slots at a time, and the job
// ranges by binary search over the slots' unit prefixes.
__device__ __noinline__ void make_plan_many(const DecodeArgs &a, DecodeSmem &S, int P, int lane, int c, int nC) {
    const int E = a.E, H = a.H, I = a.I;
    const int G = H / kGroup;
    const int pg = I / 8, pd = H / 16;
    const uint32_t ug = (uint32_t)pg * (uint32_t)G;
    int U;
    uint32_t GUB;
    // Many pairs: bitmap of the selection in shared memory, per-slot counts and a stable
    // fill of the pair lists, 32 slots per pass.
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
    U = S.U;
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
    uint32_t cts = 0;
    for (int base = 0; base < U; base += 32) {
        const int u = base + lane;
        const int n = (u < U) ? S.cnt[u] : 0;
        const uint32_t tu = (u < U) ? (uint32_t)tile_bytes(S.ubits[u]) / 64u : 0u;
        int incl = n;
        uint32_t it = tu;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, off);
            const uint32_t ot = __shfl_up_sync(0xffffffffu, it, off);
            if (lane >= off) {
                incl += o;
                it += ot;
            }
        }
        if (u < U) {
            S.pfirst[u] = carry + incl - n;
            S.cursor[u] = carry + incl - n;
            S.cgu[u] = (cts + it - tu) * ug;
            S.cd[u] = (cts + it - tu) * ug / 2u;
        }
        carry += __shfl_sync(0xffffffffu, incl, 31);
        cts += __shfl_sync(0xffffffffu, it, 31);
    }
    GUB = cts * ug;
    if (lane == 0) {
        S.pfirst[U] = carry;
        S.cgu[U] = GUB;
        S.cd[U] = GUB >> 1;
    }
    __syncwarp();
    // stable fill: pairs in ascending pair id order
    for (int base = 0; base < P; base += 32) {
        const int p = base + lane;
        const int u = (p < P) ? slot_of(S, S.sel_idx[p]) : -1 - lane;
        const uint32_t peers = __match_any_sync(0xffffffffu, u);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        if (p < P) {
            const int pos = S.cursor[u] + rank;
            S.ppair[pos] = p;
            S.ptok[pos] = (int)(((uint32_t)p * a.kmul) >> 16);
            S.pw[pos] = S.sel_w[p];
        }
        __syncwarp();
        if (p < P && rank == 0) S.cursor[u] += __popc(peers);
        __syncwarp();
    }
    const uint32_t DB = GUB >> 1, B = GUB + DB;
    int g0, g1, d0, d1;
    uint32_t mj = 0;   // largest gate/up job (units)
    for (int u = lane; u < U; u += 32) mj = max(mj, (S.cgu[u + 1] - S.cgu[u]) / pg);
    mj = __reduce_max_sync(0xffffffffu, mj);
    const bool mono = (unsigned long long)(mj + 2u) * (unsigned)nC <= DB;
    int gcut = 0;
    if (lane < 2) {
        const int cc = c + lane;
        gcut = (cc >= nC) ? U * pg : job_at_unit(S.cgu, U, pg, cut_units(a, GUB, cc, nC));
    }
    g0 = __shfl_sync(0xffffffffu, gcut, 0);
    g1 = __shfl_sync(0xffffffffu, gcut, 1);
    int dcut = 0;
    if (lane < 2) {
        const int cc = c + lane;
        const int gj = lane == 0 ? g0 : g1;
        const uint32_t pos = mono ? cut_units(a, B, cc, nC) - job_start_unit(S.cgu, U, pg, gj)
                                  : cut_units(a, DB, cc, nC);
        dcut = (cc >= nC) ? U * pd : job_at_unit(S.cd, U, pd, pos);
    }
    d0 = __shfl_sync(0xffffffffu, dcut, 0);
    d1 = __shfl_sync(0xffffffffu, dcut, 1);
    if (lane == 0) {
        S.g0 = g0;
        S.g1 = g1;
        S.d0 = d0;
        S.d1 = d1;
        S.nGU = g1 - g0;
    }
    __syncwarp();
}

// The plan, by one warp: unique experts in ascending id (slots), each slot's pair list in
// ascending pair id (token-major, so ascending token), unit prefixes of the gate/up and down
// job sequences, and this CTA's job ranges. P = 0 (an aborted routing) gives an empty plan.
// A 64-byte unit is the granule of the job sequences: a tile of `bits` is tile_bytes(bits) / 64
// units, a gate/up job G tiles and a down job GI tiles, so that an expert's down units are
// exactly half its gate/up units.
__device__ void make_plan(const DecodeArgs &a, DecodeSmem &S, int P, int lane, int c, int nC) {
    if (P > 32) {
        make_plan_many(a, S, P, lane, c, nC);
        return;
    }
    const int H = a.H, I = a.I;
    const int G = H / kGroup, GI = I / kGroup;
    const int pg = I / 8, pd = H / 16;
    const uint32_t ug = (uint32_t)pg * (uint32_t)G;   // gate/up units of an expert per unit of tile size
    int U;
    uint32_t GUB;                      // gate/up units of all slots
    uint32_t lo, hi, ts;               // slot lanes: the slot's gate/up units [lo, hi), units per tile
    int slot;                          // slot of the lane's expert
    bool slot_lane;                    // the lane holds the first pair of its expert
    uint32_t mts;                      // largest units per tile over the slots
    bool uniform;                      // every slot has the same tile size (all jobs alike)
    {
        // One pair per lane. Each lane counts, over a packed list of all pairs {expert, units
        // per tile, first pair of its expert}, the distinct experts below its own (its slot),
        // their units and the pairs below it; the totals come out of the same pass.
        const bool v = lane < P;
        const int e = v ? S.sel_idx[lane] : 0;
        const float pw = v ? S.sel_w[lane] : 0.f;
        const int eb = S.ebits[e];
        const uint32_t eo = S.eoff[e];
        const uint32_t tsl = (uint32_t)tile_bytes(eb) / 64u;
        uint32_t same = 1u << lane;   // one token: its experts are distinct
        if (a.T > 1) same = __match_any_sync(0xffffffffu, v ? e : -1 - lane);
        const int rank = __popc(same & ((1u << lane) - 1u));
        const bool first = v && rank == 0;
        // entries past P: an id above every expert, no units, not first
        S.plist[lane] = v ? ((uint32_t)e | (tsl << 16) | (first ? 0x80000000u : 0u)) : 0xFFFFu;
        __syncwarp();
        uint32_t nsl = 0, units = 0, pbelow = 0, nU = 0, tot = 0, mtsmin = 0xFFFFu;
        mts = 0;
        const uint4 *pl = reinterpret_cast<const uint4 *>(S.plist);
        for (int q4 = 0; q4 < (P + 3) / 4; ++q4) {
            const uint4 w4 = pl[q4];
            const uint32_t ws[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t w = ws[j];
                const bool lt = (w & 0xFFFFu) < (uint32_t)e;
                const uint32_t tq = (w >> 31) ? (w >> 16) & 0x7FFFu : 0u;   // units of a first entry
                pbelow += lt ? 1u : 0u;
                nsl += (lt && tq) ? 1u : 0u;
                units += lt ? tq : 0u;
                nU += tq ? 1u : 0u;
                tot += tq;
                mts = max(mts, tq);
                mtsmin = min(mtsmin, tq ? tq : 0xFFFFu);
            }
        }
        U = (int)nU;
        uniform = mts == mtsmin;
        slot = (int)nsl;
        slot_lane = first;
        ts = tsl;
        lo = units * ug;
        hi = lo + tsl * ug;
        GUB = tot * ug;
        if (first) {
            S.ubits[slot] = eb;
            S.uoff[slot] = eo;
            S.pfirst[slot] = (int)pbelow;
            S.cgu[slot] = lo;
            S.cd[slot] = lo >> 1;
        }
        if (v) {
            const int pos = (int)pbelow + rank;
            S.ppair[pos] = lane;
            S.ptok[pos] = (int)(((uint32_t)lane * a.kmul) >> 16);
            S.pw[pos] = pw;
        }
        if (lane == 0) {
            S.U = U;
            S.pfirst[U] = P;
            S.cgu[U] = GUB;
            S.cd[U] = GUB >> 1;
        }
    }
    // Job ranges. The gate/up sequence is cut at multiples of its units / nCTA; the down
    // sequence is cut so that each CTA's gate/up + down units are the layer's units / nCTA. That
    // cut is monotone in the CTA index when every CTA's down share exceeds one gate/up job (plus
    // rounding); otherwise (tiny layers) the down sequence is cut on its own.
    const uint32_t DB = GUB >> 1, B = GUB + DB;
    int g0, g1, d0, d1;
    {
        const uint32_t jbg = ts * (uint32_t)G, jbd = ts * (uint32_t)GI;   // units per job of the lane's slot
        const uint32_t mj = mts * (uint32_t)G;                            // largest gate/up job
        const bool mono = (unsigned long long)(mj + 2u) * (unsigned)nC <= DB;
        uint32_t st0, st1, unused;
        if (uniform && U > 0) {
            // all jobs of a sequence alike: the first job at or after q is ceil(q / job units)
            const uint32_t ug1 = mts * (uint32_t)G, ud1 = mts * (uint32_t)GI;
            const int NG = U * pg, ND = U * pd;
            g0 = min(NG, (int)ceil_div_small(cut_units(a, GUB, c, nC), ug1));
            g1 = (c + 1 < nC) ? min(NG, (int)ceil_div_small(cut_units(a, GUB, c + 1, nC), ug1)) : NG;
            const uint32_t q0 = mono ? cut_units(a, B, c, nC) - (uint32_t)g0 * ug1 : cut_units(a, DB, c, nC);
            const uint32_t q1 = mono ? cut_units(a, B, c + 1, nC) - (uint32_t)g1 * ug1 : cut_units(a, DB, c + 1, nC);
            d0 = min(ND, (int)ceil_div_small(q0, ud1));
            d1 = (c + 1 < nC) ? min(ND, (int)ceil_div_small(q1, ud1)) : ND;
        } else {
        g0 = job_at_unit_warp(lo, hi, jbg, slot, slot_lane, pg, U, cut_units(a, GUB, c, nC), GUB, st0);
        if (c + 1 < nC) {
            g1 = job_at_unit_warp(lo, hi, jbg, slot, slot_lane, pg, U, cut_units(a, GUB, c + 1, nC), GUB, st1);
        } else {
            g1 = U * pg;
            st1 = GUB;
        }
        const uint32_t q0 = mono ? cut_units(a, B, c, nC) - st0 : cut_units(a, DB, c, nC);
        d0 = job_at_unit_warp(lo >> 1, hi >> 1, jbd, slot, slot_lane, pd, U, q0, DB, unused);
        if (c + 1 < nC) {
            const uint32_t q1 = mono ? cut_units(a, B, c + 1, nC) - st1 : cut_units(a, DB, c + 1, nC);
            d1 = job_at_unit_warp(lo >> 1, hi >> 1, jbd, slot, slot_lane, pd, U, q1, DB, unused);
        } else {
            d1 = U * pd;
        }
        }
    }
    if (lane == 0) {
        S.g0 = g0;
        S.g1 = g1;
        S.d0 = d0;
        S.d1 = d1;
        S.nGU = g1 - g0;
    }
    __syncwarp();
}

// ------------------------------------------------------------------------------ finalisation
// Gate/up job gj: SiLU-GLU of the slot's sums (rows 0-7 gate, 8-15 up of intermediate rows
// 8 rb .. 8 rb + 7), h stored as a bf16 pair hi + lo (exact to about 2^-17 relative); the
// slot is cleared for its next job.
template <int NT>
__device__ __forceinline__ void finalize_gu(const DecodeArgs &a, const DecodeSmem &S, int gj, float *slot, int lane) {
    const int pg = a.I / 8;
    const int u = gj / pg, rb = gj % pg;
    const int pf = S.pfirst[u], nu = S.pfirst[u + 1] - pf;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        float *sp = slot + nt * 128 + lane;
        const float gate[2] = {sp[0], sp[32]}, up[2] = {sp[64], sp[96]};
        sp[0] = sp[32] = sp[64] = sp[96] = 0.f;
#pragma unroll
        for (int col = 0; col < 2; ++col) {
            const int q = nt * 8 + 2 * t + col;
            if (q < nu) {
                const float h = __fdividef(gate[col], 1.f + __expf(-gate[col])) * up[col];
                const __nv_bfloat16 hi = __float2bfloat16_rn(h);
                const __nv_bfloat16 lo = __float2bfloat16_rn(h - __bfloat162float(hi));
                const size_t o = (size_t)S.ppair[pf + q] * a.I + rb * 8 + g;
                a.h_hi[o] = __bfloat16_as_ushort(hi);
                a.h_lo[o] = __bfloat16_as_ushort(lo);
            }
        }
    }

}
// Down job dj, computed whole by one warp: w * y of rows 16 rb + g and 16 rb + g + 8 added into
// the fp32 output accumulator.
// Down job dj, summed in one warp's registers: w * y added into the fp32 output accumulator.
template <int NT>
__device__ __forceinline__ void finalize_down(const DecodeArgs &a, const DecodeSmem &S, int dj, const float (&acc)[NT][4],
                                              const float (&acc2)[NT][4], int lane) {
    const int pd = a.H / 16;
    const int u = dj / pd, rb = dj % pd;
    const int pf = S.pfirst[u], nu = S.pfirst[u + 1] - pf;
    const int g = lane >> 2, t = lane & 3;
    const int row = rb * 16 + g;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int col = 0; col < 2; ++col) {
            const int q = nt * 8 + 2 * t + col;
            if (q < nu) {
                float *o = a.out_acc + (size_t)S.ptok[pf + q] * a.H + row;
                const float wgt = S.pw[pf + q];
                red_add_f32(o, wgt * (acc[nt][col] + acc2[nt][col]));
                red_add_f32(o + 8, wgt * (acc[nt][2 + col] + acc2[nt][2 + col]));
            }
        }
    }
}

// ------------------------------------------------------------------------------ kernel
template <int NT>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeArgs a, const DecodeLayout L) {
    extern __shared__ __align__(128) uint8_t dyn[];
    DecodeSmem &S = *reinterpret_cast<DecodeSmem *>(dyn);
    uint8_t *act = dyn + L.act;
    float *accs = reinterpret_cast<float *>(dyn + L.accs);
    float *Xs = reinterpret_cast<float *>(dyn + L.xs);
    uint8_t *ring = dyn + L.ring;
    constexpr int NSLOT = slots_for<NT>();
    constexpr int SF = slot_floats<NT>();
    const int NS = L.stages;
    const int T = a.T, H = a.H, I = a.I, E = a.E, K = a.k, P = T * K;
    const int G = H / kGroup, GI = I / kGroup;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nC = gridDim.x, c = blockIdx.x;
    uint32_t *status = &a.ctl->status;
    const bool xs_on = (size_t)T * H * 2 <= (size_t)kActBytes;
    const uint16_t *xsm = reinterpret_cast<const uint16_t *>(act);
    const int ne = (E > c) ? (E - c + nC - 1) / nC : 0;   // router rows of this CTA: c, c+nC, ...
    const bool wr_on = (size_t)ne * H * 4 <= (size_t)NS * kStageBytes;
    const float *wsm = reinterpret_cast<const float *>(ring);

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
        S.is_last = 0;
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
    for (int i = threadIdx.x; i < NSLOT * SF; i += kThreads) accs[i] = 0.f;
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
            bulk_g2s(smem_u32(act), a.x, bytes, smem_u32(&S.xbar));
        }
        S.epoch = *reinterpret_cast<volatile unsigned long long *>(&a.ctl->done) / (unsigned long long)nC;
    }
    if (xs_on && !mbar_wait(smem_u32(&S.xbar), 0, a.wait_ns, status)) S.abort = 1;
    if (wr_on && ne > 0 && !mbar_wait(smem_u32(&S.wbar), 0, a.wait_ns, status)) S.abort = 1;
    __syncthreads();
    const unsigned long long epoch = S.epoch;
    const uint32_t tag = (uint32_t)(epoch + 1ull);
    const uint16_t *xr = xs_on ? xsm : a.x;
    // The CTA's ne * T dot products over H. With fewer of them than warps each is split into
    // slices of whole 256-element strides, one slice per warp, and the slices' sums are added
    // in slice order.
    // Every logit word goes to lrep copies of the T x E block (lstride words apart, spread over
    // the L2 slices); CTA c polls copy c mod lrep, so that no slice serves all CTAs' polls.
    auto row_bias = [&](int i, int e) -> float { return i < kBiasRows ? S.bias[i] : (a.bias ? a.bias[e] : 0.f); };
    auto publish_logit = [&](int t, int e, float l) {
        const unsigned long long w = ((unsigned long long)tag << 32) | (unsigned long long)__float_as_uint(l);
        for (int r = 0; r < a.lrep; ++r) st_relaxed_u64(a.logits + (size_t)r * a.lstride + (size_t)t * E + e, w);
    };
    const int nq = ne * T;
    const int nstr = (H + 255) / 256;
    const int nsl = (nq > 0 && nq < kWarps) ? min(kWarps / nq, nstr) : 1;
    for (int it = warp; it < nq * nsl; it += kWarps) {
        const int q = it / nsl, sl = it - q * nsl;
        const int i = q / T, t = q % T;
        const int e = c + i * nC;
        const float *wrow = wr_on ? wsm + (size_t)i * H : a.wr + (size_t)e * H;
        const uint16_t *xrow = xr + (size_t)t * H;
        const int h1 = min(H, (sl + 1) * nstr / nsl * 256);
        float acc0 = 0.f, acc1 = 0.f;
        for (int h = sl * nstr / nsl * 256 + lane * 8; h < h1; h += 256) {
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
        if (lane == 0) {
            if (nsl == 1) publish_logit(t, e, acc + row_bias(i, e));
            else S.lpart[it] = acc;
        }
    }
    if (nsl > 1) {
        __syncthreads();
        if (threadIdx.x < nq) {
            const int q = threadIdx.x, i = q / T, t = q % T;
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
        const bool ok = !S.abort && (E <= 256 ? token_topk(a, S, t, tag, lane, c) : token_topk_wide(a, S, t, tag, lane, c));
        if (!ok && lane == 0) S.abort = 1;
    };
    // tokens go to warps from the control warp on, so that with one token the control warp routes
    // it and makes the plan without a CTA barrier in between
    for (int t = (warp + 1) % kWarps; t < T; t += kWarps) route_token(t);
    if (warp != kCW || T > 1) group_sums(threadIdx.x, T > 1 ? kThreads : kCW * 32);
    if (T > 1) __syncthreads();
    if (warp == kCW) {
        __syncwarp();
        make_plan(a, S, S.abort ? 0 : P, lane, c, nC);
        __syncwarp();
        // hand the plan to the consumer warps and start streaming without waiting for them
        plan_ready_arrive();
        // ------------------------------------------------------------ producer (one thread)
        if (lane != 0) return;
        uint32_t cc = 0;
        bool ok = true;
        const bool has_down = S.d1 > S.d0;
        for (int ph = 0; ph < 2 && ok; ++ph) {
            const bool gu = ph == 0;
            const int jend = gu ? S.g1 : S.d1;
            for (int j = gu ? S.g0 : S.d0; j < jend && ok;) {
                const Region r = region_at(S, a, gu, j);
                const int nch = region_chunks(r, gu ? chunk_jobs<NT>() : kStageBytes);
                const int jnext = j + r.tiles / r.tpj;
                for (int ch = 0; ch < nch; ++ch) {
                    int c0, m;
                    chunk_range(r, nch, ch, c0, m);
                    const int s = cc % NS;
                    const uint32_t use = cc / NS;
                    if (use > 0 && (S.abort || !mbar_wait(smem_u32(&S.empty[s]), (use - 1) & 1u, a.wait_ns, status))) {
                        S.abort = 1;
                        ok = false;
                        break;
                    }
                    // the chunk's descriptor, published to the consumers by the barrier's arrival
                    const int jlo = c0 / r.tpj, jhi = (c0 + m - 1) / r.tpj;
                    ChunkDesc dd;
                    dd.job0 = r.jg0 + jlo;
                    dd.base_off = (jlo * r.tpj - c0) * r.tb;
                    dd.njobs = (short)(jhi - jlo + 1);
                    dd.k0 = (short)(c0 - jlo * r.tpj);
                    dd.k1 = (short)(c0 + m - jhi * r.tpj);
                    dd.tpj = (short)r.tpj;
                    dd.tb = (unsigned short)r.tb;
                    dd.bits = (unsigned char)r.bits;
                    const bool last = ch == nch - 1 && jnext >= jend && (!gu || !has_down);
                    dd.flags = (unsigned char)((gu ? 1 : 0) | (last ? 2 : 0));
                    dd.u = (short)r.u;
                    dd.pad = 0;
                    S.desc[s] = dd;
                    const uint32_t bytes = (uint32_t)(m * r.tb);
                    const uint32_t fb = smem_u32(&S.full[s]);
                    mbar_expect_tx(fb, bytes);
                    bulk_g2s(smem_u32(ring + (size_t)s * kStageBytes), r.src + (size_t)c0 * r.tb, bytes, fb);
                    ++cc;
                }
                j = jnext;
            }
        }
        // copies still in flight land before the CTA may exit
        for (uint32_t q = cc > (uint32_t)NS ? cc - NS : 0; q < cc; ++q)
            mbar_wait(smem_u32(&S.full[q % NS]), (q / NS) & 1u, a.wait_ns, status);
        return;
    }

    // ---------------------------------------------------------------- consumers
    plan_ready_wait();
    const int g = lane >> 2, t = lane & 3;
    float acc[NT][4], acc2[NT][4];
    auto zero_acc = [&]() {
#pragma unroll
        for (int i = 0; i < NT; ++i) {
            acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
            acc2[i][0] = acc2[i][1] = acc2[i][2] = acc2[i][3] = 0.f;
        }
    };
    JobCtx<NT> jc;
    bool hfit = true;
    const uint16_t *hh = nullptr, *hl = nullptr;
    const float *hs = nullptr;

    // h of expert slot u into shared memory (with its per-group sums), after the expert's
    // gate/up rows are published by every CTA that computed some; all consumer warps take part.
    // This CTA's gate/up rows are all stored (their finalisers passed a consumer barrier since):
    // one fence makes them visible GPU-wide, then each expert's counter grows by the CTA's jobs.
    bool published = false;
    auto publish_h = [&]() {
        if (threadIdx.x == 0 && !published && S.g1 > S.g0) {
            __threadfence();
            const int pg = I / 8;
            const int u0 = S.g0 / pg, u1 = (S.g1 - 1) / pg;
            for (int u = u0; u <= u1; ++u)
                atomicAdd(&a.h_ready[u], (uint32_t)(min(S.g1, (u + 1) * pg) - max(S.g0, u * pg)));
        }
        published = true;
    };
    auto load_h = [&](int u) {
        consumer_sync();   // nobody still reads the previous contents of act
        if (!S.abort) publish_h();
        if (threadIdx.x == 0 && !S.abort &&
            !wait_counter(&a.h_ready[u], (uint32_t)(I / 8), a.wait_ns, status))
            S.abort = 1;
        consumer_sync();
        const int pf = S.pfirst[u], nu = S.pfirst[u + 1] - pf;
        const size_t hsb = align_up((size_t)nu * GI * 4, 16), hb = (size_t)nu * I * 2;
        hfit = hsb + 2 * hb <= (size_t)kActBytes;
        float *hsw = reinterpret_cast<float *>(act);
        uint16_t *hhw = reinterpret_cast<uint16_t *>(act + hsb), *hlw = hhw + (size_t)nu * I;
        if (!S.abort) {
            // eight threads per group of 64 values: one 16-byte piece of h hi and of h lo each,
            // the group's sum over a 3-step shuffle
            const int n8 = nu * GI * 8;
            for (int base = threadIdx.x - lane; base < n8; base += kCW * 32) {
                const int i8 = base + lane;
                const bool v = i8 < n8;
                const int item = i8 >> 3, part = i8 & 7;
                const int q = item / GI, grp = item - q * GI;
                uint4 vh = make_uint4(0, 0, 0, 0), vl = make_uint4(0, 0, 0, 0);
                if (v) {
                    const size_t o = (size_t)S.ppair[pf + q] * I + (size_t)grp * kGroup + part * 8;
                    vh = __ldcg(reinterpret_cast<const uint4 *>(a.h_hi + o));
                    vl = __ldcg(reinterpret_cast<const uint4 *>(a.h_lo + o));
                }
                const uint32_t w8[8] = {vh.x, vh.y, vh.z, vh.w, vl.x, vl.y, vl.z, vl.w};
                float sum = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) sum += __uint_as_float(w8[j] << 16) + __uint_as_float(w8[j] & 0xFFFF0000u);
                sum += __shfl_xor_sync(0xffffffffu, sum, 1);
                sum += __shfl_xor_sync(0xffffffffu, sum, 2);
                sum += __shfl_xor_sync(0xffffffffu, sum, 4);
                if (v && part == 0) hsw[item] = sum;
                if (v && hfit) {
                    const size_t d = (size_t)q * I + (size_t)grp * kGroup + part * 8;
                    *reinterpret_cast<uint4 *>(hhw + d) = vh;
                    *reinterpret_cast<uint4 *>(hlw + d) = vl;
                }
            }
        }
        consumer_sync();
        hs = hsw;
        hh = hhw;
        hl = hlw;
    };
    auto set_ctx = [&](int u, bool gu) {
        const int pf = S.pfirst[u];
        const int nu = S.pfirst[u + 1] - pf;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int q = nt * 8 + g, q0 = nt * 8 + 2 * t, q1 = q0 + 1;
            jc.has[nt] = q < nu;
            jc.has0[nt] = q0 < nu;
            jc.has1[nt] = q1 < nu;
            const int qq = q < nu ? q : 0, qq0 = q0 < nu ? q0 : 0, qq1 = q1 < nu ? q1 : 0;
            if (gu) {
                const int tok = S.ptok[pf + qq];
                jc.b[nt] = a.x + (size_t)tok * H;
                jc.b2[nt] = nullptr;
                jc.sb[nt] = smem_u32(xsm) + (uint32_t)(tok * H * 2);
                jc.sb2[nt] = 0;
                jc.xs0[nt] = smem_u32(Xs) + (uint32_t)(S.ptok[pf + qq0] * G * 4);
                jc.xs1[nt] = smem_u32(Xs) + (uint32_t)(S.ptok[pf + qq1] * G * 4);
            } else {
                jc.b[nt] = a.h_hi + (size_t)S.ppair[pf + qq] * I;
                jc.b2[nt] = a.h_lo + (size_t)S.ppair[pf + qq] * I;
                jc.sb[nt] = smem_u32(hh) + (uint32_t)(qq * I * 2);
                jc.sb2[nt] = smem_u32(hl) + (uint32_t)(qq * I * 2);
                jc.xs0[nt] = smem_u32(hs) + (uint32_t)(qq0 * GI * 4);
                jc.xs1[nt] = smem_u32(hs) + (uint32_t)(qq1 * GI * 4);
            }
        }
        jc.bg = gu ? !xs_on : !hfit;
    };
    // Gate/up jobs are split along K: tile k of a job goes to warp k % kCW, which adds its partial
    // sums into the job's slot (CTA-local job q uses slot q % NSLOT) after its last tile of the
    // job. A down job (a few tiles) belongs to one warp and is finalised from its registers.
    auto add_partial = [&](int q) {
        float *sp = accs + (q % NSLOT) * SF;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) red_shared_f32(sp + (nt * 4 + i) * 32 + lane, acc[nt][i] + acc2[nt][i]);
        zero_acc();
    };
    // Gate/up jobs fj0 .. fj0 + fn - 1 have all their partials in their slots (after the barrier
    // that follows the chunk that completed them); warp gj % kCW finalises job gj.
    int fj0 = 0, fn = 0;
    auto finalize_pending = [&]() {
        for (int i = 0; i < fn; ++i) {
            const int gj = fj0 + i;
            if (gj % kCW == warp) finalize_gu<NT>(a, S, gj, accs + ((gj - S.g0) % NSLOT) * SF, lane);
        }
        fn = 0;
    };

    zero_acc();
    int s = 0;
    uint32_t par = 0;
    int cur_u = -1, cur_gu = -1, tpj = 1, kl = -1;
    bool more = S.g1 > S.g0 || S.d1 > S.d0;
    while (more) {
        const bool got = !S.abort && mbar_wait(smem_u32(&S.full[s]), par, a.wait_ns, status);
        // One barrier per chunk: every warp's partials of the previous chunk are in, and all
        // warps take the same abort decision.
        if (consumer_sync_or(!got || S.abort)) {
            if (lane == 0) S.abort = 1;
            break;
        }
        finalize_pending();
        const ChunkDesc d = S.desc[s];
        const bool gu = d.flags & 1;
        if (d.u != cur_u || (int)gu != cur_gu) {
            if (!gu) load_h(d.u);
            set_ctx(d.u, gu);
            cur_u = d.u;
            cur_gu = gu;
            tpj = d.tpj;
            kl = (warp < tpj) ? warp + kCW * ((tpj - 1 - warp) / kCW) : -1;   // this warp's last tile of a job
        }
        const uint8_t *sb = ring + (size_t)s * kStageBytes + d.base_off;
        for (int i = 0; i < d.njobs; ++i) {
            const int k0 = i == 0 ? d.k0 : 0, k1 = i == d.njobs - 1 ? d.k1 : tpj;
            const uint8_t *job_base = sb + (size_t)i * tpj * d.tb;
            const int gj = d.job0 + i;
            if (gu) {
                if (d.bits == 4) run_tiles<4, NT, true>(job_base, d.tb, k0, k1, warp, jc, lane, acc, acc2);
                else if (d.bits == 6) run_tiles<6, NT, true>(job_base, d.tb, k0, k1, warp, jc, lane, acc, acc2);
                else run_tiles<8, NT, true>(job_base, d.tb, k0, k1, warp, jc, lane, acc, acc2);
                if (kl >= k0 && kl < k1) add_partial(gj - S.g0);
            } else if ((gj - S.d0) % kCW == warp) {
                if (d.bits == 4) run_tiles_seq<4, NT>(job_base, d.tb, k0, k1, jc, lane, acc, acc2);
                else if (d.bits == 6) run_tiles_seq<6, NT>(job_base, d.tb, k0, k1, jc, lane, acc, acc2);
                else run_tiles_seq<8, NT>(job_base, d.tb, k0, k1, jc, lane, acc, acc2);
                if (k1 == tpj) {
                    finalize_down<NT>(a, S, gj, acc, acc2, lane);
                    zero_acc();
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&S.empty[s]));
        fj0 = d.job0;
        fn = gu ? d.njobs - (d.k1 < tpj ? 1 : 0) : 0;
        more = !(d.flags & 2);
        if (++s == NS) {
            s = 0;
            par ^= 1u;
        }
    }
    if (!consumer_sync_or(S.abort)) {
        finalize_pending();
        if (!published) {
            // no down job here: the gate/up rows are published after their finalisers are done
            consumer_sync();
            publish_h();
        }
    }

    // ---------------------------------------------------------------- completion
    consumer_sync();
    if (threadIdx.x == 0) {
        // release (this CTA's additions, ordered before it by the barrier) and acquire (the
        // other CTAs' additions, for the last CTA) in one step
        const unsigned long long old = atom_add_acq_rel_u64(&a.ctl->done, 1ull);
        S.is_last = (old + 1ull == (epoch + 1ull) * (unsigned long long)nC) ? 1 : 0;
    }
    consumer_sync();
    if (S.is_last) {
        // every CTA's additions are complete: convert, then leave the accumulator and the
        // readiness counters zero for the next call
        float4 *acc4 = reinterpret_cast<float4 *>(a.out_acc);
        uint2 *out4 = reinterpret_cast<uint2 *>(a.out);
        for (int i = threadIdx.x; i < T * H / 4; i += kCW * 32) {
            const float4 v = __ldcg(acc4 + i);
            const __nv_bfloat162 lo2 = __floats2bfloat162_rn(v.x, v.y), hi2 = __floats2bfloat162_rn(v.z, v.w);
            out4[i] = make_uint2(*reinterpret_cast<const uint32_t *>(&lo2), *reinterpret_cast<const uint32_t *>(&hi2));
            __stcg(acc4 + i, make_float4(0.f, 0.f, 0.f, 0.f));
        }
        for (int i = threadIdx.x; i < kMaxP; i += kCW * 32) a.h_ready[i] = 0u;
    }
}

// Copies of the exchanged logit words within the fixed logit region (kMaxT x kMaxE words): the
// T x E block at 4 KB-aligned strides, up to 32 copies.
void logit_copies(int T, int E, int &rep, int &stride) {
    stride = (int)align_up((size_t)T * E, 512);
    rep = 1;
    while (rep < 32 && (size_t)(rep * 2) * stride <= (size_t)kMaxT * kMaxE) rep *= 2;
}

template <int NT>
moe_status_t launch_nt(const DecodeArgs &a, const DeviceInfo *dev, cudaStream_t st) {
    const DecodeLayout L = decode_layout<NT>(a.T, a.H, dev->max_smem_optin);
    if (L.stages < 2) return MOE_ERR_UNSUPPORTED;
    static bool attr_set[64] = {false};
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64) return MOE_ERR_CUDA;
    if (!attr_set[d]) {
        if (cudaFuncSetAttribute(decode_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dev->max_smem_optin) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_set[d] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(dev->sms);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, decode_kernel<NT>, a, L) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

}  // namespace

moe_status_t launch_decode(const uint16_t *x, const float *wr, const float *bias, const void *packed,
                           int T, int H, int I, int E, int k, uint16_t *out, int32_t *idx_out,
                           float *w_out, void *ws, cudaStream_t st) {
    // (I bound: the per-group sums of one expert's h must fit the activation region)
    if (T * k > kMaxP || T > kMaxT || H > kDecodeMaxH || I > 16384) return MOE_ERR_UNSUPPORTED;
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
    a.h_ready = reinterpret_cast<uint32_t *>(w8 + W.h_ready);
    a.out_acc = reinterpret_cast<float *>(w8 + W.out_acc);
    a.h_hi = reinterpret_cast<uint16_t *>(w8 + W.h_hi);
    a.h_lo = reinterpret_cast<uint16_t *>(w8 + W.h_lo);
    a.wait_ns = wait_limit_ns();
    a.rnC = 1.0 / (double)dev->sms;
    {
        // Granlund-Montgomery constants for division by the number of CTAs
        const uint32_t d = (uint32_t)dev->sms;
        uint32_t l = 0;
        while ((1ull << l) < d) ++l;   // ceil(log2 d)
        a.cm = (uint32_t)(((1ull << 32) * ((1ull << l) - d)) / d + 1ull);
        a.cs1 = l < 1 ? l : 1u;
        a.cs2 = l > 0 ? l - 1u : 0u;
    }
    a.kmul = (uint32_t)((65536 + k - 1) / k);
    logit_copies(T, E, a.lrep, a.lstride);
    if (T <= 8) return launch_nt<1>(a, dev, st);
    if (T <= 16) return launch_nt<2>(a, dev, st);
    return launch_nt<4>(a, dev, st);
}

}  // namespace moe
