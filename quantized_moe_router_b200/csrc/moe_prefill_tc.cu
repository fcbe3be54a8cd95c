// moe_prefill_tc.cu -- the prefill grouped GEMMs on the 5th-generation tensor cores (tcgen05).
//
// In prefill the expert block is a dense contraction: after bucketing, expert e multiplies its
// n_e tokens (about 128 at 4096 tokens, 256 experts, top-8) by its dequantised weights, and a
// long prompt touches nearly every expert of a layer (the pages "Qwen-tin" and
// "--moe-direct-io"). Both GEMMs run as one persistent kernel each (one CTA per SM) whose work
// unit is (expert, 128 weight rows, up to 256 of the expert's tokens):
//   * 1 producer warp streams the unit's packed tiles from HBM into a ring of raw slots with 1-D
//     bulk copies (one per row block and K chunk of up to 4 tiles; the copy engine, not the
//     load/store path, so the token-row loads below do not queue behind the weight stream);
//   * 8 dequantiser warps, one of the unit's 8 row blocks each per K step (measured slightly
//     faster than 4 warps of two row blocks; the dequantisation runs at the SMs' issue rate, so
//     more warps add little), read their packed 16x64 tiles from the raw slot and write
//     w = (q - z) * s as fp16 into a 128-byte-swizzled K-major tile A [128 x 64];
//   * 1 loader thread brings the unit's token rows into a swizzled tile B [N x 64] with 2-D tensor
//     copies (TMA, 64 rows each, the 128-byte swizzle applied by the copy engine): gate/up reads
//     x16, the pairs' hidden states in bucket order as fp16 (scaled per token by a power of two
//     so that no value overflows), down reads h16 (fp16, scaled per pair);
//   * 1 warp issues tcgen05.mma (kind::f16, fp16 x fp16 -> fp32, M = 128, N = tokens rounded up
//     to 16) into one of two TMEM accumulators, 4 MMAs (K = 16) per 64-wide K step, and frees
//     each ring stage with tcgen05.commit;
//   * 8 epilogue warps (two per TMEM lane quarter, taking alternate 32-column chunks) read the
//     other accumulator with tcgen05.ld while the next unit runs: gate/up undoes the token scale,
//     pairs each gate row with its up row (8 TMEM lanes apart), applies SiLU-GLU and stores h as
//     fp16 with one power-of-two exponent per 16 columns (a small kernel between the GEMMs brings
//     each pair's h to one common exponent); down undoes the pair's exponent and adds w * y into
//     the fp32 output accumulator with red.add. The per-column tables of the next unit (token,
//     scale) are loaded while the current unit is processed.
// fp16 operands (11-bit significands) keep the block within its error bound where bf16
// operands (8-bit) would not; every scaling is by a power of two and exact.
// Every mbarrier wait is bounded; the CTA frees its TMEM before it exits.
#include <atomic>
#include <mutex>

#include "moe_tc.cuh"

namespace moe {

namespace {

constexpr int kTM = 128;                          // weight rows per unit (UMMA M)
constexpr int kMaxN = 256;                        // tokens per unit (UMMA N limit)
constexpr int kABStages = 3;
constexpr int kABytes = kTM * 128;                // 128 rows x 64 fp16
constexpr int kMaxRaw = 8;                        // raw ring slots (K chunks) at most
constexpr int kDnSkew = 128;                      // extra bytes per down K step in a raw slot (3 x 32 used)
#ifndef MOE_TC_DQ_WARPS
#define MOE_TC_DQ_WARPS 8
#endif
constexpr int kDqWarps = MOE_TC_DQ_WARPS, kLdWarps = 1;
constexpr int kBPW = 8 / kDqWarps;                // 16-row blocks of the A tile per dequantiser warp
constexpr int kRowBox = 64;                       // token rows per tensor copy
constexpr int kMmaWarp = kDqWarps + kLdWarps;
constexpr int kEpiWarps = 8;                      // two per TMEM lane quarter
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kEpiWarp0 = kMmaWarp + 1;
constexpr int kProdWarp = kEpiWarp0 + kEpiWarps;
constexpr int kTcWarps = kProdWarp + 1;
constexpr int kTcThreads = kTcWarps * 32;
constexpr uint32_t kTmemCols = 2 * kMaxN;         // two accumulators of 256 fp32 columns
constexpr int kBarEpi = 1;                        // named barrier of the epilogue warps (0 is __syncthreads)
constexpr int kMaxSub = 64;                       // 16-column blocks of a down row (I <= 1024)
static_assert(kEpiThreads == kMaxN, "one epilogue thread per column of a unit");

struct TcArgs {
    const uint8_t *packed;
    int H, I, E;
    const int32_t *nt_start, *pair_tok;
    const int4 *ntab;      // N tiles: {expert | bits << 16, first row in the bucket, rows, bucket offset}
    const float *pscale;   // per pair in bucket order: gate/up 2^xexp of its token, down w * 2^fexp
    uint16_t *h;           // gate/up output: h16
    int8_t *hexp_out;      // gate/up output: exponents of h16
    float *out_acc;        // down output: [T x H] fp32
    int smem_bytes;        // dynamic shared memory of the launch
    uint64_t wait_ns;
    uint32_t *status;
};

struct TcShared {
    uint64_t ab_full[kABStages];
    uint64_t ab_empty[kABStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t fin;
    uint64_t raw_full[kMaxRaw];
    uint64_t raw_empty[kMaxRaw];
    uint32_t tmem_base;
    volatile int abort;
};

// ------------------------------------------------------------------------------ work units
// An expert's n tokens are cut into ceil(n / 256) N tiles of equal size (rounded up to 16).
__host__ __device__ inline int ntile_size(int n) {
    const int c = (n + kMaxN - 1) / kMaxN;
    return c == 0 ? 0 : (((n + c - 1) / c + 15) & ~15);
}
__host__ __device__ inline int ntile_count(int n) {
    const int s = ntile_size(n);
    return s == 0 ? 0 : (n + s - 1) / s;
}

struct Unit {
    int e, bits, mt, n0, nn, nr, base;
};

// Unit u = (N tile u / mtiles, M tile u % mtiles), read from the N-tile table.
__device__ __forceinline__ Unit unit_at(const TcArgs &a, int u, int mtiles) {
    Unit U;
    const int ti = u / mtiles;
    U.mt = u - ti * mtiles;
    const int4 v = __ldg(a.ntab + ti);
    U.e = v.x & 0xFFFF;
    U.bits = v.x >> 16;
    U.n0 = v.y;
    U.nn = v.z;
    U.nr = (v.z + 15) & ~15;
    U.base = v.w;
    return U;
}

// Bounded mbarrier wait that also gives up when another role of the CTA has aborted.
__device__ __forceinline__ bool tc_wait(TcShared &S, const TcArgs &a, uint64_t *bar, uint32_t parity) {
    const uint32_t b = smem_u32(bar);
    if (mbar_try_wait(b, parity)) return true;
    const uint64_t t0 = global_timer();
    while (true) {
        if (mbar_try_wait_sleep(b, parity, 20000u)) return true;
        if (S.abort) return false;
        if (global_timer() - t0 > a.wait_ns) {
            atomicOr(a.status, kStatusTimeout);
            S.abort = 1;
            return false;
        }
    }
}

// 2^e as fp32 for |e| <= 126
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((e + 127) << 23); }
// the exponent f with 2^14 <= max|v| * 2^-f < 2^15 (0 when max|v| is 0), from the bits of max|v|
__device__ __forceinline__ int scale_exp(float vmax) {
    const uint32_t b = __float_as_uint(vmax);
    if (b == 0u) return 0;
    const int e = (int)((b >> 23) & 0xFF) - 127;
    return max(-100, min(100, e - 14));
}

// ------------------------------------------------------------------------------ dequantisation
// A code nibble becomes an fp32 value by byte placement (prmt) under a fixed exponent byte:
//   low nibble q of byte x  -> 0x3F0q0000 = 0.5 + q/256   (row g of the lane fragment)
//   high nibble q of byte x -> 0x3F80(q<<4)00 = 1 + q/2048 (row g+8)
// so w = (q - z) * s = f * S + C with S = 256 s (2048 s) and C = -(128 + z) s (-(2048 + z) s).
// C is rounded once to fp32 (|error| <= 2^-24 |C|, far below the fp16 rounding of w). (Measured
// on B200: this fp32 form beats an fp16x2 s*q form with the zero point folded into extra K steps.)
__device__ __forceinline__ float nib_float(uint32_t m, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(m), "r"(0x3F800000u), "r"(sel));
    return __uint_as_float(r);
}
// (x0 * S + C, x1 * S + C) with one packed fp32x2 FMA, rounded to an fp16 pair (x0 in the low half)
__device__ __forceinline__ uint32_t fma2_h(float x0, float x1, float S, float C) {
    const float2 r = __ffma2_rn(make_float2(x0, x1), make_float2(S, S), make_float2(C, C));
    const __half2 v = __floats2half2_rn(r.x, r.y);
    return *reinterpret_cast<const uint32_t *>(&v);
}
// x * S + y * S2 + C for two elements (6/8-bit codes: the low and the high code plane)
__device__ __forceinline__ uint32_t fma2_h_hi(float x0, float x1, float y0, float y1, float S, float S2, float C) {
    float t0 = fmaf(x0, S, C), t1 = fmaf(x1, S, C);
    t0 = fmaf(y0, S2, t0);
    t1 = fmaf(y1, S2, t1);
    const __half2 v = __floats2half2_rn(t0, t1);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// The 16 values of row g (cols 16t .. 16t+15) and of row g+8 of one 16x64 tile, stored as fp16
// into the swizzled A tile rows 16b+g and 16b+g+8. lo16: the lane's 16 lo-plane bytes; hip: its
// hi-plane bytes (8-bit: 16 bytes in the lo arrangement; 6-bit: the tile's two hi words, or, with
// DQ, the four half-words of the down layout, one per MMA); szp: its scale/zero entry (8 bytes).
// Word j of the lo bytes holds columns 16t+4j+{0,1,2,3} in bytes {0,2,1,3}: row g in the low
// nibbles, row g+8 in the high nibbles.
template <int BITS, bool DQ>
__device__ __forceinline__ void dequant_fragment(const uint8_t *lo16, const uint8_t *hip, const uint8_t *szp, int L,
                                                 uint8_t *As, int b) {
    const int g = L >> 2, t = L & 3;
    const uint4 lo = *reinterpret_cast<const uint4 *>(lo16);
    const uint2 sz = *reinterpret_cast<const uint2 *>(szp);
    const float sA = half_lo(sz.x), zA = half_hi(sz.x), sB = half_lo(sz.y), zB = half_hi(sz.y);
    const uint32_t w[4] = {lo.x, lo.y, lo.z, lo.w};
    uint32_t ra[8], rb[8];
    if (BITS == 4) {
        const float SA = 256.f * sA, CA = -(128.f + zA) * sA;
        const float SB = 2048.f * sB, CB = -(2048.f + zB) * sB;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t m0 = w[j] & 0x0F0F0F0Fu, m1 = w[j] & 0xF0F0F0F0u;
            ra[2 * j] = fma2_h(nib_float(m0, 0x7054), nib_float(m0, 0x7254), SA, CA);
            ra[2 * j + 1] = fma2_h(nib_float(m0, 0x7154), nib_float(m0, 0x7354), SA, CA);
            rb[2 * j] = fma2_h(nib_float(m1, 0x7604), nib_float(m1, 0x7624), SB, CB);
            rb[2 * j + 1] = fma2_h(nib_float(m1, 0x7614), nib_float(m1, 0x7634), SB, CB);
        }
    } else if (BITS == 8) {
        // q = lo + 16 hi, the hi plane in the same nibble arrangement
        const uint4 hi = *reinterpret_cast<const uint4 *>(hip);
        const uint32_t v[4] = {hi.x, hi.y, hi.z, hi.w};
        const float SA = 256.f * sA, SA2 = 4096.f * sA, CA = -(128.f + 2048.f + zA) * sA;
        const float SB = 2048.f * sB, SB2 = 32768.f * sB, CB = -(2048.f + 32768.f + zB) * sB;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t m0 = w[j] & 0x0F0F0F0Fu, m1 = w[j] & 0xF0F0F0F0u;
            const uint32_t h0 = v[j] & 0x0F0F0F0Fu, h1 = v[j] & 0xF0F0F0F0u;
            ra[2 * j] = fma2_h_hi(nib_float(m0, 0x7054), nib_float(m0, 0x7254), nib_float(h0, 0x7054),
                                  nib_float(h0, 0x7254), SA, SA2, CA);
            ra[2 * j + 1] = fma2_h_hi(nib_float(m0, 0x7154), nib_float(m0, 0x7354), nib_float(h0, 0x7154),
                                      nib_float(h0, 0x7354), SA, SA2, CA);
            rb[2 * j] = fma2_h_hi(nib_float(m1, 0x7604), nib_float(m1, 0x7624), nib_float(h1, 0x7604),
                                  nib_float(h1, 0x7624), SB, SB2, CB);
            rb[2 * j + 1] = fma2_h_hi(nib_float(m1, 0x7614), nib_float(m1, 0x7634), nib_float(h1, 0x7614),
                                      nib_float(h1, 0x7634), SB, SB2, CB);
        }
    } else {
        // 6-bit: q = lo + 16 hi, hi in 2-bit fields (word j/2, pair s = 4(j&1) + r at bits 2s and
        // 16 + 2s; r = 0: row g cols +0/+1, 1: row g+8 cols +0/+1, 2: row g +2/+3, 3: row g+8 +2/+3)
        uint2 hi = *reinterpret_cast<const uint2 *>(hip);
        if (DQ) {
            // half-words {MMA 0, 1} and {MMA 2, 3} -> the tile's hi words (bytes lo0 lo1 hi0 hi1)
            hi.x = __byte_perm(hi.x, 0u, 0x3120);
            hi.y = __byte_perm(hi.y, 0u, 0x3120);
        }
        const float SA = 256.f * sA, SA2 = 16.f * sA, CA = -(128.f + zA) * sA;
        const float SB = 2048.f * sB, SB2 = 16.f * sB, CB = -(2048.f + zB) * sB;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t m0 = w[j] & 0x0F0F0F0Fu, m1 = w[j] & 0xF0F0F0F0u;
            const uint32_t hv = (j < 2) ? hi.x : hi.y;
            const int s0 = 8 * (j & 1);
            auto f2 = [&](int sh) { return (float)((hv >> sh) & 3u); };
            ra[2 * j] = fma2_h_hi(nib_float(m0, 0x7054), nib_float(m0, 0x7254), f2(s0), f2(16 + s0), SA, SA2, CA);
            ra[2 * j + 1] = fma2_h_hi(nib_float(m0, 0x7154), nib_float(m0, 0x7354), f2(s0 + 4), f2(20 + s0), SA,
                                      SA2, CA);
            rb[2 * j] = fma2_h_hi(nib_float(m1, 0x7604), nib_float(m1, 0x7624), f2(s0 + 2), f2(18 + s0), SB, SB2,
                                  CB);
            rb[2 * j + 1] = fma2_h_hi(nib_float(m1, 0x7614), nib_float(m1, 0x7634), f2(s0 + 6), f2(22 + s0), SB,
                                      SB2, CB);
        }
    }
    const int r0 = 16 * b + g, r1 = r0 + 8;
    *reinterpret_cast<uint4 *>(As + sw128_off(r0, 2 * t)) = make_uint4(ra[0], ra[1], ra[2], ra[3]);
    *reinterpret_cast<uint4 *>(As + sw128_off(r0, 2 * t + 1)) = make_uint4(ra[4], ra[5], ra[6], ra[7]);
    *reinterpret_cast<uint4 *>(As + sw128_off(r1, 2 * t)) = make_uint4(rb[0], rb[1], rb[2], rb[3]);
    *reinterpret_cast<uint4 *>(As + sw128_off(r1, 2 * t + 1)) = make_uint4(rb[4], rb[5], rb[6], rb[7]);
}

template <bool GU>
struct Geometry {
    int K, KG, mtiles, nrb;
    size_t skip_tiles;  // tiles of an expert stored before this matrix's tiles
    __device__ explicit Geometry(const TcArgs &a) {
        K = GU ? a.H : a.I;
        KG = K / kGroup;
        nrb = GU ? a.I / 8 : a.H / 16;  // 16-row blocks of the matrix
        mtiles = (nrb + 7) / 8;
        skip_tiles = GU ? 0 : gu_tiles(a.H, a.I);
    }
};

// 2^d as an fp16 pair for d <= 0 (subnormal below 2^-14, zero below 2^-24)
__device__ __forceinline__ uint32_t h2_pow2(int d) {
    uint32_t b = 0;
    if (d >= -14) b = (uint32_t)(15 + d) << 10;
    else if (d >= -24) b = 1u << (24 + d);
    return b | (b << 16);
}
__device__ __forceinline__ uint32_t hmul2_bits(uint32_t a, uint32_t b) {
    __half2 r = __hmul2(*reinterpret_cast<const __half2 *>(&a), *reinterpret_cast<const __half2 *>(&b));
    return *reinterpret_cast<const uint32_t *>(&r);
}

// ------------------------------------------------------------------------------ the kernel
template <bool GU>
__global__ void __launch_bounds__(kTcThreads, 1) tc_grouped_kernel(const TcArgs a, const __grid_constant__ CUtensorMap tmap) {
    extern __shared__ uint8_t tc_dyn[];
    __shared__ TcShared S;
    __shared__ __align__(16) int ep_i[2][kMaxN];     // epilogue: token of each column (down)
    __shared__ __align__(16) float ep_f[2][kMaxN];   // epilogue: scale of each column
    const uint32_t pad = (1024u - (smem_u32(tc_dyn) & 1023u)) & 1023u;
    uint8_t *base = tc_dyn + pad;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Geometry<GU> G(a);
    const int nunits = __ldg(a.nt_start + a.E) * G.mtiles;
    const int nr_max = __ldg(a.nt_start + a.E + 1);
    const int SUB = a.I / 16;                                  // 16-column blocks of an h row
    // shared memory: kABStages x [A 16 KB | B nr_max x 128 B], then the h staging tile (gate/up),
    // then the raw ring
    const uint32_t bbytes = (uint32_t)align_up((size_t)(nr_max > 0 ? nr_max : 16), kRowBox) * 128;
    const uint32_t stage_bytes = kABytes + bbytes;
    uint8_t *ring = base;
    uint8_t *side = ring + (size_t)kABStages * stage_bytes;
    const uint32_t side_bytes = GU ? (uint32_t)align_up((size_t)nr_max * 128, 1024) : 0u;
    uint8_t *raw = side + side_bytes;
    // K chunks of KC tiles per row block (KC divides the unit's K steps, so chunks never straddle
    // units); a raw slot holds one chunk of the 8 row blocks at the layer's widest tile. The
    // largest KC that leaves room for 3 slots (at least 2).
    const int tb_max = __ldg(a.nt_start + a.E + 2);
    const long long raw_room = (long long)a.smem_bytes - (long long)pad - (long long)(raw - base);
    // a down K step in a slot: scale/zero entries, then the four quarters, quarter q shifted by
    // 32 q bytes so that the lanes (g, t) reading quarter t fall into distinct shared-memory banks
    const int kstep = GU ? 8 * tb_max : 8 * tb_max + kDnSkew;
    int KC = 1, R = 0;
    for (int kc = 4; kc >= 1; kc >>= 1) {
        if (G.KG % kc) continue;
        const int r = (int)(raw_room / ((long long)kc * kstep));
        if (r >= 3 || kc == 1) {
            KC = kc;
            R = r;
            break;
        }
    }
    R = R > kMaxRaw ? kMaxRaw : R;
    const uint32_t slot_bytes = (uint32_t)(KC * kstep);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kABStages; ++s) {
            mbar_init(smem_u32(&S.ab_full[s]), kDqWarps + 1);
            mbar_init(smem_u32(&S.ab_empty[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&S.acc_full[s]), 1);
            mbar_init(smem_u32(&S.acc_empty[s]), kEpiWarps);
        }
        mbar_init(smem_u32(&S.fin), 1);
        for (int s = 0; s < kMaxRaw; ++s) {
            mbar_init(smem_u32(&S.raw_full[s]), 1);
            mbar_init(smem_u32(&S.raw_empty[s]), kDqWarps);
        }
        S.abort = (R < 2) ? 1 : 0;
        if (R < 2) atomicOr(a.status, kStatusCheck);
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S.tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const bool run = !S.abort;

    if (warp < kDqWarps) {
        // ------------------------------------------------------------ dequantisers
        bool ok = run;
        // step counters kept incrementally (no division in the loop): position jk in the K
        // chunk, raw slot rs and its phase, A/B stage slot and its phase
        int jk = 0, rs = 0, slot = 0;
        uint32_t rpar = 0, apar = 0;
        bool first_pass = true;
        for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
            const Unit U = unit_at(a, u, G.mtiles);
            // per unit: the expert's width and whether this warp's row block exists
            const int bits = U.bits;
            const int tb = tile_bytes(bits);
            // this warp's row blocks warp + kDqWarps * i, and whether they exist in this M tile
            bool have_all = true;
#pragma unroll
            for (int i = 0; i < kBPW; ++i) have_all &= 8 * U.mt + warp + kDqWarps * i < G.nrb;
            for (int kg = 0; kg < G.KG; ++kg) {
                if (jk == 0 && !tc_wait(S, a, &S.raw_full[rs], rpar)) {
                    ok = false;
                    break;
                }
                if (!first_pass && !tc_wait(S, a, &S.ab_empty[slot], apar ^ 1u)) {
                    ok = false;
                    break;
                }
                uint8_t *As = ring + (size_t)slot * stage_bytes;
                // the lane's lo / hi / scale-zero bytes of row block b of this K step: gate/up
                // slots hold [row block][K chunk] tiles; down slots hold per K step the scale/zero
                // entries of the unit's super-tiles and its four quarters
                auto frag = [&](int b, const uint8_t *&lo16, const uint8_t *&hip, const uint8_t *&szp) {
                    if (GU) {
                        // slot: per row-block pair, its KC group columns x 2 tiles
                        const uint8_t *rawt =
                            raw + (size_t)rs * slot_bytes + (size_t)(((b >> 1) * KC + jk) * 2 + (b & 1)) * tb;
                        lo16 = rawt + 16 * lane;
                        hip = rawt + kLoBytes + (bits == 8 ? 16 : 8) * lane;
                        szp = rawt + kLoBytes + hi_bytes(bits) + 8 * (lane >> 2);
                    } else {
                        const int qb = d_quarter_bytes(bits), g = lane >> 2, t = lane & 3;
                        const uint8_t *base = raw + (size_t)rs * slot_bytes + (size_t)jk * (8 * tb + kDnSkew);
                        const uint8_t *qp = base + 512 + (size_t)t * (2 * qb + 32) + (size_t)(b >> 2) * qb;
                        lo16 = qp + (b & 3) * 128 + 16 * g;
                        hip = qp + kLoBytes + (b & 3) * (bits == 8 ? 128 : 64) + (bits == 8 ? 16 : 8) * g;
                        szp = base + (b >> 2) * 256 + (b & 3) * 64 + 8 * g;
                    }
                };
                if (have_all && bits == 4) {
#pragma unroll
                    for (int i = 0; i < kBPW; ++i) {
                        const uint8_t *lo16, *hip, *szp;
                        frag(warp + kDqWarps * i, lo16, hip, szp);
                        dequant_fragment<4, !GU>(lo16, hip, szp, lane, As, warp + kDqWarps * i);
                    }
                } else {
#pragma unroll 1
                    for (int i = 0; i < kBPW; ++i) {
                        const int b = warp + kDqWarps * i;
                        const uint8_t *lo16, *hip, *szp;
                        frag(b, lo16, hip, szp);
                        if (8 * U.mt + b >= G.nrb) {
                            const uint4 z = make_uint4(0, 0, 0, 0);
                            const int g = lane >> 2, t = lane & 3;
                            *reinterpret_cast<uint4 *>(As + sw128_off(16 * b + g, 2 * t)) = z;
                            *reinterpret_cast<uint4 *>(As + sw128_off(16 * b + g, 2 * t + 1)) = z;
                            *reinterpret_cast<uint4 *>(As + sw128_off(16 * b + g + 8, 2 * t)) = z;
                            *reinterpret_cast<uint4 *>(As + sw128_off(16 * b + g + 8, 2 * t + 1)) = z;
                        } else if (bits == 4) {
                            dequant_fragment<4, !GU>(lo16, hip, szp, lane, As, b);
                        } else if (bits == 8) {
                            dequant_fragment<8, !GU>(lo16, hip, szp, lane, As, b);
                        } else {
                            dequant_fragment<6, !GU>(lo16, hip, szp, lane, As, b);
                        }
                    }
                }
                fence_proxy_async();  // generic-proxy stores -> visible to the tensor core
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(smem_u32(&S.ab_full[slot]));
                    if (jk == KC - 1) mbar_arrive(smem_u32(&S.raw_empty[rs]));
                }
                if (++jk == KC) {
                    jk = 0;
                    if (++rs == R) {
                        rs = 0;
                        rpar ^= 1u;
                    }
                }
                if (++slot == kABStages) {
                    slot = 0;
                    apar ^= 1u;
                    first_pass = false;
                }
            }
        }
    } else if (warp < kMmaWarp) {
        // ------------------------------------------------------------ token-row loader (one thread)
        if (lane == 0 && run) {
            uint32_t j = 0;
            bool ok = true;
            const uint64_t tm = reinterpret_cast<uint64_t>(&tmap);
            for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
                const Unit U = unit_at(a, u, G.mtiles);
                const int nb = (U.nr + kRowBox - 1) / kRowBox;
                for (int kg = 0; kg < G.KG; ++kg, ++j) {
                    const int slot = j % kABStages;
                    const uint32_t use = j / kABStages;
                    if (use > 0 && !tc_wait(S, a, &S.ab_empty[slot], (use - 1) & 1u)) {
                        ok = false;
                        break;
                    }
                    const uint32_t Bs = smem_u32(ring + (size_t)slot * stage_bytes + kABytes);
                    const uint32_t fb = smem_u32(&S.ab_full[slot]);
                    mbar_expect_tx(fb, (uint32_t)(nb * kRowBox * 128));
                    // rows past the unit's tokens belong to the next bucket (or lie past the
                    // matrix and read as zeros); their columns are never used
                    for (int i = 0; i < nb; ++i)
                        asm volatile(
                            "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
                            ::"r"(Bs + (uint32_t)(i * kRowBox * 128)), "l"(tm), "r"(kg * kGroup),
                            "r"(U.base + U.n0 + i * kRowBox), "r"(fb)
                            : "memory");
                }
            }
            // copies still in flight land before the CTA may exit
            for (uint32_t q = j > (uint32_t)kABStages ? j - kABStages : 0; q < j; ++q)
                mbar_wait(smem_u32(&S.ab_full[q % kABStages]), (q / kABStages) & 1u, a.wait_ns, a.status);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issue
        uint32_t j = 0, i = 0;
        bool ok = run;
        for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x, ++i) {
            const Unit U = unit_at(a, u, G.mtiles);
            const uint32_t buf = i & 1u;
            if (i >= 2 && !tc_wait(S, a, &S.acc_empty[buf], ((i >> 1) - 1) & 1u)) break;
            tc_fence_after();
            const uint32_t idesc = idesc_f16_f32(kTM, U.nr);
            const uint32_t d_tmem = tmem + buf * kMaxN;
            for (int kg = 0; kg < G.KG; ++kg, ++j) {
                const int slot = j % kABStages;
                if (!tc_wait(S, a, &S.ab_full[slot], (j / kABStages) & 1u)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t As = smem_u32(ring + (size_t)slot * stage_bytes), Bs = As + kABytes;
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(d_tmem, sw128_desc(As + 32 * kk), sw128_desc(Bs + 32 * kk), idesc,
                                 (kg > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(smem_u32(&S.ab_empty[slot]));
                }
                __syncwarp();
            }
            if (!ok) break;
            if (lane == 0) umma_commit(smem_u32(&S.acc_full[buf]));
            __syncwarp();
        }
        // every MMA issued by this warp has completed once `fin` flips; waited for (bounded) even
        // after an abort, so that TMEM is released only when no MMA still writes it
        if (lane == 0) umma_commit(smem_u32(&S.fin));
        __syncwarp();
        mbar_wait(smem_u32(&S.fin), 0, a.wait_ns, a.status);
    } else if (warp == kProdWarp) {
        // ------------------------------------------------------------ weight producer (one thread)
        if (lane == 0 && run) {
            const PackedExpert *pe = reinterpret_cast<const PackedExpert *>(a.packed + sizeof(PackedHeader));
            uint32_t chunk = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
                const Unit U = unit_at(a, u, G.mtiles);
                const PackedExpert ex = pe[U.e];
                const int tb = tile_bytes(ex.bits);
                const uint8_t *mat = a.packed + ex.offset + G.skip_tiles * tb;
                const int nb = min(8, G.nrb - 8 * U.mt);   // row blocks of this M tile
                for (int k0 = 0; k0 < G.KG; k0 += KC, ++chunk) {
                    const uint32_t rs = chunk % R;
                    if (chunk >= (uint32_t)R && !tc_wait(S, a, &S.raw_empty[rs], ((chunk / R) - 1) & 1u)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&S.raw_full[rs]);
                    mbar_expect_tx(fb, (uint32_t)(nb * KC * tb));
                    uint8_t *slot = raw + (size_t)rs * slot_bytes;
                    if (GU) {
                        // one copy per row-block pair: its tiles of group columns k0 .. k0 + KC - 1
                        for (int pp = 0; pp < nb / 2; ++pp)
                            bulk_g2s(smem_u32(slot + (size_t)pp * 2 * KC * tb),
                                     mat + ((size_t)(4 * U.mt + pp) * G.KG + k0) * 2 * tb, (uint32_t)(2 * KC * tb), fb);
                    } else {
                        // per K step: the scale/zero entries of the unit's super-tiles, then its
                        // piece of each quarter (nb / 4 super-tiles from super-tile 2 * mt)
                        const int nst = nb / 4, qb = d_quarter_bytes(ex.bits);
                        for (int kk = 0; kk < KC; ++kk) {
                            const uint8_t *blk = mat + (size_t)(k0 + kk) * d_block_bytes(a.H, ex.bits);
                            uint8_t *dstk = slot + (size_t)kk * (8 * tb + kDnSkew);
                            bulk_g2s(smem_u32(dstk), blk + (size_t)2 * U.mt * 256, (uint32_t)(nst * 256), fb);
                            for (int q = 0; q < 4; ++q)
                                bulk_g2s(smem_u32(dstk + 512 + (size_t)q * (2 * qb + 32)),
                                         blk + d_quarter_offset(a.H, ex.bits, q) + (size_t)2 * U.mt * qb,
                                         (uint32_t)(nst * qb), fb);
                        }
                    }
                }
            }
            // copies still in flight land before the CTA may exit
            for (uint32_t q = chunk > (uint32_t)R ? chunk - R : 0; q < chunk; ++q)
                mbar_wait(smem_u32(&S.raw_full[q % R]), (q / R) & 1u, a.wait_ns, a.status);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                         // this warp may read TMEM lanes 32q .. 32q+31
        const int half = (warp - kEpiWarp0) >> 2;       // it takes the 32-column chunks 2c + half
        const int row = 32 * q + lane;                  // accumulator row
        const int et = threadIdx.x - kEpiWarp0 * 32;    // 0 .. kEpiThreads - 1 (= kMaxN - 1)
        uint32_t i = 0;
        bool ok = run;
        // column tables (token, scale) of unit i in buffer i & 1; those of unit i + 1 are loaded
        // into registers while unit i is processed and stored after it
        int nt_tok = 0;
        float nt_sc = 0.f;
        auto load_table = [&](const Unit &V) {
            nt_tok = 0;
            nt_sc = 0.f;
            if (et < V.nn) {
                nt_tok = __ldg(a.pair_tok + V.base + V.n0 + et);
                nt_sc = __ldg(a.pscale + V.base + V.n0 + et);
            }
        };
        Unit U{};
        if ((int)blockIdx.x < nunits) {
            U = unit_at(a, blockIdx.x, G.mtiles);
            load_table(U);
            ep_i[0][et] = nt_tok;
            ep_f[0][et] = nt_sc;
        }
        // every epilogue warp walks all units through the same named barriers; after an expired
        // wait it only skips the work
        for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++i) {
            const uint32_t buf = i & 1u;
            named_sync(kBarEpi, kEpiThreads);   // tables of unit i stored; the staging tile is free
            const int un = u + (int)gridDim.x;
            Unit Un{};
            if (un < nunits) {
                Un = unit_at(a, un, G.mtiles);
                load_table(Un);
            }
            if (ok && !tc_wait(S, a, &S.acc_full[buf], (i >> 1) & 1u)) ok = false;
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + buf * kMaxN;
            const int *tk = ep_i[buf];
            const float *tf = ep_f[buf];
            if (GU) {
                // row 16b + g: gate (g < 8) or up (g >= 8) of intermediate column 8b + (g & 7)
                const bool gate = (row & 8) == 0;
                const int col = 8 * (row >> 4) + (row & 7);
                uint16_t *stg = reinterpret_cast<uint16_t *>(side);
                // 16 columns from cb: the gate lane finishes token cb+2p, its up partner cb+2p+1
                auto glu16 = [&](const uint32_t(&v)[16], int cb) {
                    float recv[8], hv[8];
#pragma unroll
                    for (int p = 0; p < 8; ++p)
                        recv[p] = __shfl_xor_sync(0xffffffffu, __uint_as_float(gate ? v[2 * p + 1] : v[2 * p]), 8);
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        const float xs = tf[cb + 2 * p + (gate ? 0 : 1)];
                        const float gv = (gate ? __uint_as_float(v[2 * p]) : recv[p]) * xs;
                        const float uv = (gate ? recv[p] : __uint_as_float(v[2 * p + 1])) * xs;
                        hv[p] = __fdividef(gv, 1.f + __expf(-gv)) * uv;
                    }
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        const int tok = cb + 2 * p + (gate ? 0 : 1);
                        // one exponent per 16 columns of this token: the max over the 16 lanes
                        // that hold the token (gate lanes 0-7, 16-23 or up lanes 8-15, 24-31)
                        const uint32_t hb = (tok < U.nn) ? (__float_as_uint(hv[p]) & 0x7FFFFFFFu) : 0u;
                        const uint32_t mx =
                            gate ? __reduce_max_sync(0x00FF00FFu, hb) : __reduce_max_sync(0xFF00FF00u, hb);
                        const int f = scale_exp(__uint_as_float(mx));
                        stg[tok * 64 + col] = __half_as_ushort(__float2half_rn(hv[p] * exp2i(-f)));
                        if ((lane & 23) == 0 && tok < U.nn)   // lane 0 (gate group) or lane 8 (up group)
                            a.hexp_out[(size_t)(U.base + U.n0 + tok) * SUB + 4 * U.mt + q] = (int8_t)f;
                    }
                };
                for (int c0 = 32 * half; ok && c0 < U.nr; c0 += 64) {
                    uint32_t v0[16], v1[16];
                    const bool two = c0 + 16 < U.nr;
                    tmem_ld16_nowait(taddr + c0, v0);
                    if (two) tmem_ld16_nowait(taddr + c0 + 16, v1);
                    tmem_wait_ld();
                    glu16(v0, c0);
                    if (two) glu16(v1, c0 + 16);
                }
                tc_fence_before();
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(smem_u32(&S.acc_empty[buf]));
                named_sync(kBarEpi, kEpiThreads);
                // coalesced copy-out: 8 threads per 128-byte token row
                const int cc = et & 7;
                for (int tok = et >> 3; ok && tok < U.nn; tok += kEpiThreads / 8) {
                    const uint4 val = *reinterpret_cast<const uint4 *>(side + tok * 128 + cc * 16);
                    *reinterpret_cast<uint4 *>(a.h + (size_t)(U.base + U.n0 + tok) * a.I + 64 * U.mt + cc * 8) = val;
                }
            } else {
                const int orow = kTM * U.mt + row;
                const bool valid = orow < a.H;
                float *ob = a.out_acc + orow;
                auto down16 = [&](const uint32_t(&v)[16], int cb) {
                    int t16[16];
                    float s16[16];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int4 ti4 = *reinterpret_cast<const int4 *>(tk + cb + 4 * j);
                        const float4 tf4 = *reinterpret_cast<const float4 *>(tf + cb + 4 * j);
                        t16[4 * j] = ti4.x, t16[4 * j + 1] = ti4.y, t16[4 * j + 2] = ti4.z, t16[4 * j + 3] = ti4.w;
                        s16[4 * j] = tf4.x, s16[4 * j + 1] = tf4.y, s16[4 * j + 2] = tf4.z, s16[4 * j + 3] = tf4.w;
                    }
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj)
                        if (valid && cb + jj < U.nn)
                            red_add_f32_free(ob + (size_t)t16[jj] * a.H, s16[jj] * __uint_as_float(v[jj]));
                };
                for (int c0 = 32 * half; ok && c0 < U.nr; c0 += 64) {
                    uint32_t v0[16], v1[16];
                    const bool two = c0 + 16 < U.nr;
                    tmem_ld16_nowait(taddr + c0, v0);
                    if (two) tmem_ld16_nowait(taddr + c0 + 16, v1);
                    tmem_wait_ld();
                    down16(v0, c0);
                    if (two) down16(v1, c0 + 16);
                }
                tc_fence_before();
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(smem_u32(&S.acc_empty[buf]));
            }
            if (un < nunits) {
                ep_i[buf ^ 1u][et] = nt_tok;
                ep_f[buf ^ 1u][et] = nt_sc;
            }
            U = Un;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    }
}

// Exclusive prefix of the experts' N-tile counts (nt_start[E] = total), the largest N tile in
// rows (nt_start[E + 1]), the largest tile in bytes (nt_start[E + 2]) and the N-tile table; one
// CTA of 1024 threads.
__global__ void ntile_scan_kernel(const int32_t *counts, const int32_t *offsets, const uint8_t *packed, int E,
                                  int32_t *nt_start, int4 *ntab) {
    __shared__ int warp_tot[32];
    __shared__ int warp_max[32];
    __shared__ int tb_max;
    const int e = threadIdx.x, lane = e & 31, w = e >> 5;
    const PackedExpert *pe = reinterpret_cast<const PackedExpert *>(packed + sizeof(PackedHeader));
    if (e == 0) tb_max = 0;
    __syncthreads();
    if (e < E) atomicMax(&tb_max, tile_bytes(pe[e].bits));
    const int n = e < E ? counts[e] : 0;
    const int c = ntile_count(n);
    const int sz = (ntile_size(n) + 15) & ~15;
    int incl = c, mx = sz;
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    if (lane == 31) warp_tot[w] = incl;
    if (lane == 0) warp_max[w] = mx;
    __syncthreads();
    if (w == 0) {
        const int v = warp_tot[lane];
        int iv = v, m = warp_max[lane];
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, iv, off);
            if (lane >= off) iv += o;
            m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
        }
        warp_tot[lane] = iv - v;
        if (lane == 0) warp_max[0] = m;
    }
    __syncthreads();
    if (e < E) {
        const int excl = warp_tot[w] + incl - c;
        nt_start[e] = excl;
        if (e == E - 1) {
            nt_start[E] = excl + c;
            nt_start[E + 1] = warp_max[0];
        }
        const int bits = pe[e].bits, s = ntile_size(n), off = offsets[e];
        for (int j = 0; j < c; ++j) ntab[excl + j] = make_int4(e | (bits << 16), j * s, min(s, n - j * s), off);
    }
    if (e == 0) nt_start[E + 2] = tb_max;
}

// xexp[t]: the exponent that keeps every |x[t] * 2^-xexp[t]| below 2^15 (0 unless some |x| >= 2^15);
// one warp per token.
__global__ void xexp_kernel(const uint16_t *x, int T, int H, int32_t *xexp) {
    const int lane = threadIdx.x & 31;
    for (int t = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); t < T; t += gridDim.x * (blockDim.x / 32)) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * H);
        uint32_t mx = 0;
        for (int i = lane; i < H / 8; i += 32) {
            const uint4 v = __ldg(src + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) mx = max(mx, max((w[j] << 16) & 0x7FFFFFFFu, w[j] & 0x7FFF0000u));
        }
        mx = __reduce_max_sync(0xffffffffu, mx);
        const int e = (int)((mx >> 23) & 0xFF) - 127;
        if (lane == 0) xexp[t] = (mx != 0u && e >= 15) ? e - 14 : 0;
    }
}

// x16[p] = fp16(x[pair_tok[p]] * 2^-xexp[token]) for every pair p in bucket order, and the
// pair's column scale 2^xexp[token]; one warp per pair.
__global__ void x16_gather_kernel(const uint16_t *x, const int32_t *pair_tok, const int32_t *xexp, int P, int H,
                                  uint16_t *x16, float *pscale) {
    const int lane = threadIdx.x & 31;
    for (int p = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); p < P; p += gridDim.x * (blockDim.x / 32)) {
        const int t = __ldg(pair_tok + p);
        const int xe = __ldg(xexp + t);
        const float sc = exp2i(-xe);
        if (lane == 0) pscale[p] = exp2i(xe);
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * H);
        uint4 *dst = reinterpret_cast<uint4 *>(x16 + (size_t)p * H);
        for (int i = lane; i < H / 8; i += 32) {
            const uint4 v = __ldg(src + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const __half2 hv = __floats2half2_rn(__uint_as_float(w[j] << 16) * sc, __uint_as_float(w[j] & 0xFFFF0000u) * sc);
                o[j] = *reinterpret_cast<const uint32_t *>(&hv);
            }
            dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// Brings each pair's h16 to one exponent: f = max over its 16-column exponents hexp[p][*], every
// block is multiplied by 2^(hexp - f) in place (exact unless the block falls into fp16's
// subnormal range, where its contribution is negligible), and the pair's column scale for the
// down GEMM is w_p * 2^f. One warp per pair.
__global__ void h16_rescale_kernel(uint16_t *h16, const int8_t *hexp, const float *pair_w, int P, int I,
                                   float *pscale) {
    const int lane = threadIdx.x & 31;
    const int SUB = I / 16;
    for (int p = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); p < P; p += gridDim.x * (blockDim.x / 32)) {
        // the row's chunks are loaded before the exponents are reduced, so the two loads overlap
        // (8 fp16 per 16-byte chunk, two chunks per 16-column block; I <= 1024: 4 per lane)
        uint4 *row = reinterpret_cast<uint4 *>(h16 + (size_t)p * I);
        uint4 v[4];
        int eb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int ch = lane + 32 * i;
            if (ch < I / 8) {
                v[i] = row[ch];
                eb[i] = (int)hexp[(size_t)p * SUB + ch / 2];
            } else {
                eb[i] = -128;
            }
        }
        int m = max(max(eb[0], eb[1]), max(eb[2], eb[3]));
        m = __reduce_max_sync(0xffffffffu, m);
        if (lane == 0) pscale[p] = __ldg(pair_w + p) * exp2i(m);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int ch = lane + 32 * i;
            const int d = eb[i] - m;
            if (ch < I / 8 && d != 0) {
                const uint32_t f = h2_pow2(d);
                v[i].x = hmul2_bits(v[i].x, f);
                v[i].y = hmul2_bits(v[i].y, f);
                v[i].z = hmul2_bits(v[i].z, f);
                v[i].w = hmul2_bits(v[i].w, f);
                row[ch] = v[i];
            }
        }
    }
}

// 2-D tensor map of a row-major fp16 matrix [rows x cols] read in boxes of 64 columns by kRowBox rows
bool make_row_map(CUtensorMap *map, const void *base, int rows, int cols) {
    return make_tmap_2d_16(map, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, rows, cols, kRowBox);
}

template <bool GU>
moe_status_t launch_tc(const TcArgs &a0, const CUtensorMap &map, const DeviceInfo *dev, cudaStream_t st) {
    TcArgs a = a0;
    a.smem_bytes = dev->max_smem_optin - (int)sizeof(TcShared) - 4 * kMaxN * 4 - 256;
    // the attribute is per device: set once per device, race-free across host threads
    static std::once_flag once[64];
    static std::atomic<int> attr_err[64];
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64) return MOE_ERR_CUDA;
    std::call_once(once[d], [&]() {
        attr_err[d] = cudaFuncSetAttribute(tc_grouped_kernel<GU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           a.smem_bytes) != cudaSuccess;
    });
    if (attr_err[d]) return MOE_ERR_CUDA;
    tc_grouped_kernel<GU><<<(unsigned)dev->sms, kTcThreads, a.smem_bytes, st>>>(a, map);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

moe_status_t launch_tc_prefill_gemms(const uint8_t *packed, int T, int H, int I, int E, int k, const int32_t *counts,
                                     const int32_t *offsets, int32_t *nt_start, int4 *ntab, const int32_t *pair_tok,
                                     const float *pair_w, float *pscale, const uint16_t *x, uint16_t *x16,
                                     int32_t *xexp, uint16_t *h16, int8_t *hexp, float *out_acc, uint32_t *status,
                                     cudaStream_t st) {
    const DeviceInfo *dev = device_info();
    if (dev == nullptr) return MOE_ERR_CUDA;
    if (I / 16 > kMaxSub) return MOE_ERR_UNSUPPORTED;
    const size_t P = (size_t)T * k;
    CUtensorMap xmap, hmap;
    if (!make_row_map(&xmap, x16, (int)P, H) || !make_row_map(&hmap, h16, (int)P, I)) return MOE_ERR_CUDA;
    ntile_scan_kernel<<<1, 1024, 0, st>>>(counts, offsets, packed, E, nt_start, ntab);
    xexp_kernel<<<(unsigned)((T + 7) / 8 < 4096 ? (T + 7) / 8 : 4096), 256, 0, st>>>(x, T, H, xexp);
    x16_gather_kernel<<<(unsigned)((P + 7) / 8 < 8192 ? (P + 7) / 8 : 8192), 256, 0, st>>>(x, pair_tok, xexp, (int)P,
                                                                                           H, x16, pscale);
    TcArgs a{};
    a.packed = packed;
    a.H = H;
    a.I = I;
    a.E = E;
    a.nt_start = nt_start;
    a.ntab = ntab;
    a.pair_tok = pair_tok;
    a.pscale = pscale;
    a.h = h16;
    a.hexp_out = hexp;
    a.out_acc = out_acc;
    a.wait_ns = wait_limit_ns();
    a.status = status;
    moe_status_t s = launch_tc<true>(a, xmap, dev, st);
    if (s != MOE_OK) return s;
    h16_rescale_kernel<<<(unsigned)((P + 7) / 8 < 8192 ? (P + 7) / 8 : 8192), 256, 0, st>>>(h16, hexp, pair_w, (int)P,
                                                                                            I, pscale);
    s = launch_tc<false>(a, hmap, dev, st);
    if (s != MOE_OK) return s;
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
