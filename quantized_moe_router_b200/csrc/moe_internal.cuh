// moe_internal.cuh -- layouts and device helpers shared by the library's kernels.
//
// Packed expert layout (written by moe_pack_layer, read by the decode and prefill kernels).
// An expert is its gate/up part followed by its down part.
//
// Gate/up ("GU") tiles: 16 rows x 64 input columns (one quantisation group); rows 0-7 are gate
// rows 8rb..8rb+7, rows 8-15 the up rows with the same indices, so one tile holds both
// projections of eight intermediate rows; tile (rb, kg) for rb < I/8, kg < H/64. Row blocks pair
// up (2i, 2i + 1: the 16 intermediate rows 16i..16i+15) and a pair's tiles are stored K-major,
// tile (rb, kg) at ((rb / 2) * (H/64) + kg) * 2 + rb % 2, so that the gate/up tiles of 16
// intermediate rows are one contiguous run and the two tiles of each group column are adjacent. A tile is [lo nibble plane 512 B][hi plane: 0 B
// (4-bit), 256 B (6-bit), 512 B (8-bit)][scale/zero 64 B]. Lane L of a warp (g = L/4, t = L%4)
// owns bytes 16L..16L+15 of the lo plane: word j (j = 0..3) holds the eight codes that lane feeds
// to MMA j as its A operand (rows g and g+8, group columns 16t+4j .. 16t+4j+3), arranged so that
// shifting the word right by 0, 4, 8, 12 and masking 0x000F000F yields the four bf16x2 operand
// registers directly (column c+0 in bits 0/4, c+1 in 16/20, c+2 in 8/12, c+3 in 24/28; row g in
// the lower nibble of each pair). The hi plane holds code >> 4 (8-bit: the same nibble
// arrangement; 6-bit: 2-bit fields, 16 per word, pair s of word m at bits 2s and 16+2s feeding
// MMA 2m + s/4, register s%4). The scale/zero block is 8 entries of 8 bytes: entry g =
// {s(row g), z(row g), s(row g+8), z(row g+8)} as fp16.
//
// Down ("D") part: Wd [H x I] in blocks of one group column kg (64 input columns), block kg at
// kg * (H/16) * tile_bytes. Rows are taken in super-tiles of 64 (four 16-row blocks r = 0..3) and
// the group's 64 columns in four quarters of 16 (quarter q = columns 16q..16q+15), so that the
// 16 columns of one quarter are contiguous for all H rows:
//   [scale/zero: H/64 super-tiles x 256 B: super-tile st, block r, entry g (8 B) =
//                {s, z of row 64st+16r+g, s, z of row 64st+16r+g+8}]
//   [quarter 0][quarter 1][quarter 2][quarter 3], each H/64 super-tiles x qbytes(bits), where a
//   super-tile's quarter is [lo: 4 blocks r x 32 lanes x 4 B][hi: 8-bit 4 x 32 x 4 B,
//   6-bit 4 x 32 x 2 B]. Word (r, lane g,t) of quarter q holds rows 64st+16r+g and +8, columns
//   16q + 4t + {0,1,2,3} in the nibble arrangement above, i.e. it is word j = t of lane (g, q) of
//   the 16x64 tile of those rows; its 6-bit hi half-word holds the two bytes of that tile's 6-bit
//   hi plane that feed MMA j = t (bits 8(j%2).. and 16+8(j%2).. of word j/2) as its low and high
//   byte.
// One quarter across all rows is therefore the down half of a decode work unit (16 intermediate
// rows), and the four 16-byte pieces {r, lanes 4g..4g+3} of the four quarters are exactly lane
// (g, t)'s 16 lo bytes of the 16x64 tile, which is how prefill reads them.
// Packed layer = header (32 B) + E expert entries (16 B) + expert data (256-B aligned).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "moe.h"

namespace moe {

constexpr int kGroup = 64;
constexpr int kLoBytes = 512;
constexpr int kSzBytes = 64;
constexpr uint32_t kPackedMagic = 0x50454F4Du;  // "MOEP"
constexpr uint32_t kPackedVersion = 2;
constexpr int kMaxT = 32;                       // decode token limit
constexpr int kMaxK = 32;
constexpr int kMaxE = 1024;
constexpr int kMaxPairs = kMaxT * kMaxK;

__host__ __device__ constexpr int hi_bytes(int bits) { return bits == 4 ? 0 : (bits == 6 ? 256 : 512); }
__host__ __device__ constexpr int tile_bytes(int bits) { return kLoBytes + hi_bytes(bits) + kSzBytes; }

struct PackedHeader {
    uint32_t magic, version;
    int32_t E, H, I;
    uint32_t reserved[3];
};
struct PackedExpert {
    uint64_t offset;  // bytes from the start of the packed layer
    int32_t bits;
    int32_t reserved;
};
static_assert(sizeof(PackedHeader) == 32, "header size");
static_assert(sizeof(PackedExpert) == 16, "entry size");

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
__host__ __device__ inline size_t gu_tiles(int H, int I) { return (size_t)(I / 8) * (H / kGroup); }
__host__ __device__ inline size_t d_tiles(int H, int I) { return (size_t)(H / 16) * (I / kGroup); }
__host__ __device__ inline size_t expert_bytes(int H, int I, int bits) {
    return (gu_tiles(H, I) + d_tiles(H, I)) * tile_bytes(bits);
}
// down part: bytes of one group-column block, of one super-tile's quarter, and the offset of
// quarter q within a block
__host__ __device__ inline size_t d_block_bytes(int H, int bits) { return (size_t)(H / 16) * tile_bytes(bits); }
__host__ __device__ constexpr int d_quarter_bytes(int bits) { return kLoBytes + hi_bytes(bits); }
__host__ __device__ inline size_t d_quarter_offset(int H, int bits, int q) {
    return (size_t)4 * H + (size_t)q * (H / 64) * d_quarter_bytes(bits);
}
__host__ __device__ inline size_t packed_data_start(int E) {
    return align_up(sizeof(PackedHeader) + (size_t)E * sizeof(PackedExpert), 256);
}

// ------------------------------------------------------------------------------------------
// Workspace: [control 256 B][regions...], every region 256-B aligned.
struct Control {
    unsigned long long done;   // decode CTAs that have finished a call, ever (epoch = done / CTAs)
    uint32_t status;           // device status bits (kStatus*)
    uint32_t pad[61];
};
static_assert(sizeof(Control) == 256, "control block size");
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusCheck = 2u;
constexpr int kDecodeMaxP = 256;   // decode limit on T*k

// Decode workspace, fixed regions only, so that one workspace serves decode calls of any shape:
// logits, kMaxT x kMaxE 8-byte words {fp32 logit bits (low word), call tag (high word)} (a call
// writes entry t * E + e of each of its copies of the T x E block); rowcnt, one 64-bit counter per
// 256 output rows (kDecodeMaxH / 256), each grown by every CTA once per call, so that the CTA that
// completes a row group converts it; out_acc, fp32 [T x H] (up to kMaxT x kDecodeMaxH), zero
// between calls (each row group is cleared by the CTA that converts it).
constexpr int kDecodeMaxH = 8192;
constexpr int kRowGroup = 256;
struct DecodeWs {
    size_t logits, rowcnt, out_acc, total;
};
inline DecodeWs decode_ws_layout(int T, int H, int I, int E, int k) {
    (void)T;
    (void)H;
    (void)I;
    (void)E;
    (void)k;
    DecodeWs w;
    size_t o = 256;
    auto take = [&](size_t b) { size_t r = o; o = align_up(o + b, 256); return r; };
    w.logits = take((size_t)kMaxT * kMaxE * 8);
    w.rowcnt = take((size_t)(kDecodeMaxH / kRowGroup) * 8);
    w.out_acc = take((size_t)kMaxT * kDecodeMaxH * 4);
    w.total = o;
    return w;
}

// Prefill workspace. x16: the hidden states of every (token, expert) pair in bucket order as fp16
// scaled by 2^-xexp[t] per token; h: fp16 h of
// every (token, expert) pair in bucket order, scaled by 2^-hexp per 16-column block; nt_start: N-tile prefix of the experts ([E] = total, [E+1] = the
// largest N tile, rows rounded to 16); ntab: one entry per N tile {expert | bits << 16, first
// bucket row, rows, expert's bucket offset}; pscale: a per-pair column scale in bucket order
// (gate/up: 2^xexp of the pair's token; down: routing weight * 2^fexp).
struct PrefillWs {
    size_t idx, w, counts, offsets, blockhist, pair_tok, pair_w, nt_start, ntab, pscale, x16, xexp, h, hexp, out_acc,
        planes, lg, total;
    int nblk;  // token blocks of the stable scatter
};
constexpr int kScatterTokens = 64;
inline PrefillWs prefill_ws_layout(int T, int H, int I, int E, int k) {
    PrefillWs w;
    size_t o = 256;
    auto take = [&](size_t b) { size_t r = o; o = align_up(o + b, 256); return r; };
    const size_t P = (size_t)T * k;
    w.nblk = (T + kScatterTokens - 1) / kScatterTokens;
    w.idx = take(P * 4);
    w.w = take(P * 4);
    w.counts = take((size_t)E * 4);
    w.offsets = take((size_t)(E + 1) * 4);
    w.blockhist = take((size_t)w.nblk * E * 4);
    w.pair_tok = take(P * 4);
    w.pair_w = take(P * 4);
    w.nt_start = take((size_t)(E + 3) * 4);
    w.ntab = take((P / 256 + (size_t)E + 1) * 16);   // sum over experts of ceil(n_e / 256)
    w.pscale = take(P * 4);
    w.x16 = take(P * H * 2);
    w.xexp = take((size_t)T * 4);
    w.h = take(P * I * 2);
    w.hexp = take(P * (I / 16));
    w.out_acc = take((size_t)T * H * 4);
    w.planes = take((size_t)3 * E * H * 2);   // router rows as three bf16 planes
    w.lg = take((size_t)T * E * 4);           // fp32 router logits
    w.total = o;
    return w;
}

// ------------------------------------------------------------------------------------------
// Device helpers (inline PTX).
#ifdef __CUDACC__
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint64_t global_timer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// try_wait with a suspend-time hint: the thread sleeps (issuing nothing) until the phase
// completes or about `hint_ns` pass, instead of spinning
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait on an mbarrier phase. Returns false (and sets the status word) on timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                          uint32_t *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_timer() - t0 > limit_ns) {
            atomicOr(status, kStatusTimeout);
            return false;
        }
    }
}
// The same bounded wait, suspending the thread between checks (try_wait with a time hint), so that
// waiting warps take no issue slots from the warps that work.
__device__ __forceinline__ bool mbar_wait_idle(uint32_t bar, uint32_t parity, uint64_t limit_ns, uint32_t *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, 1000u)) return true;
        if (global_timer() - t0 > limit_ns) {
            atomicOr(status, kStatusTimeout);
            return false;
        }
    }
}
// 1-D bulk copy global -> shared, completion counted on an mbarrier (no multicast).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t *p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ void red_add_f32(float *p, float v) {
    asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}
// the same reduction without a compiler memory barrier, for accumulators that the issuing kernel
// never reads: loads around it may be scheduled freely
__device__ __forceinline__ void red_add_f32_free(float *p, float v) {
    asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" ::"l"(p), "f"(v));
}
// bf16x2 operand from a code word: (word >> shift) & mask | bf16(128) in both halves, i.e.
// the bf16 pair {128 + field_lo, 128 + field_hi}; exact for fields < 128.
template <uint32_t MASK>
__device__ __forceinline__ uint32_t code_pair(uint32_t w, int shift) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w >> shift), "n"(MASK), "n"(0x43004300u));
    return r;
}
// D += A(16x16 bf16, row) * B(16x8 bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t bf16x2_mul16(uint32_t v) {
    // exact multiplication of both bf16 halves by 16
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162 *>(&v);
    __nv_bfloat162 r = __hmul2(h, __floats2bfloat162_rn(16.f, 16.f));
    return *reinterpret_cast<uint32_t *>(&r);
}
__device__ __forceinline__ float half_lo(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v & 0xFFFF))); }
__device__ __forceinline__ float half_hi(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v >> 16))); }
__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

// One 16x64 tile against one n-tile of 8 columns: the MMAs of the group and the group's
// affine correction. `lo`/`hi` are the lane's code words (see the layout above), `b` the
// lane's B operand words for the group (b[2j], b[2j+1] feed MMA j) and `b2` a second B operand
// accumulated into the same sums (or nullptr). Adds s*(acc - (off + z)*X) to out[4], where
// X0/X1 are the group sums of the lane's two accumulator columns.
template <int BITS>
__device__ __forceinline__ void tile_group_mma(const uint4 &lo, const uint4 &hi, const uint2 &hi6,
                                               const uint32_t (&b)[8], const uint32_t *b2,
                                               float sA, float zA, float sB, float zB, float X0,
                                               float X1, float (&out)[4]) {
    // two independent accumulator chains (even / odd MMAs, or the hi / lo B operand) so that
    // consecutive MMAs of one warp do not wait on each other
    float c[4] = {0.f, 0.f, 0.f, 0.f}, d[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t low[4] = {lo.x, lo.y, lo.z, lo.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t w = low[j];
        const uint32_t a0 = code_pair<0x000F000Fu>(w, 0), a1 = code_pair<0x000F000Fu>(w, 4);
        const uint32_t a2 = code_pair<0x000F000Fu>(w, 8), a3 = code_pair<0x000F000Fu>(w, 12);
        if (b2) {
            mma_bf16(c, a0, a1, a2, a3, b[2 * j], b[2 * j + 1]);
            mma_bf16(d, a0, a1, a2, a3, b2[2 * j], b2[2 * j + 1]);
        } else {
            mma_bf16((j & 1) ? d : c, a0, a1, a2, a3, b[2 * j], b[2 * j + 1]);
        }
    }
    if (BITS != 4) {
        uint32_t b16[8], b216[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            b16[i] = bf16x2_mul16(b[i]);
            if (b2) b216[i] = bf16x2_mul16(b2[i]);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t a0, a1, a2, a3;
            if (BITS == 8) {
                const uint32_t w = (j == 0) ? hi.x : (j == 1) ? hi.y : (j == 2) ? hi.z : hi.w;
                a0 = code_pair<0x000F000Fu>(w, 0);
                a1 = code_pair<0x000F000Fu>(w, 4);
                a2 = code_pair<0x000F000Fu>(w, 8);
                a3 = code_pair<0x000F000Fu>(w, 12);
            } else {
                const uint32_t w = (j < 2) ? hi6.x : hi6.y;
                const int s0 = (j & 1) * 8;
                a0 = code_pair<0x00030003u>(w, s0 + 0);
                a1 = code_pair<0x00030003u>(w, s0 + 2);
                a2 = code_pair<0x00030003u>(w, s0 + 4);
                a3 = code_pair<0x00030003u>(w, s0 + 6);
            }
            if (b2) {
                mma_bf16(c, a0, a1, a2, a3, b16[2 * j], b16[2 * j + 1]);
                mma_bf16(d, a0, a1, a2, a3, b216[2 * j], b216[2 * j + 1]);
            } else {
                mma_bf16((j & 1) ? d : c, a0, a1, a2, a3, b16[2 * j], b16[2 * j + 1]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] += d[i];
    const float off = (BITS == 4) ? 128.f : 2176.f;  // 128 per plane, the hi plane weighted 16x
    out[0] += sA * (c[0] - (off + zA) * X0);
    out[1] += sA * (c[1] - (off + zA) * X1);
    out[2] += sB * (c[2] - (off + zB) * X0);
    out[3] += sB * (c[3] - (off + zB) * X1);
}
#endif  // __CUDACC__

// Host-side launch helpers (defined in moe_api.cu).
struct DeviceInfo {
    int sms;
    int cc_major, cc_minor;
    int max_smem_optin;
};
const DeviceInfo *device_info();
// MOE_OK on an sm_100 device, MOE_ERR_UNSUPPORTED on another, MOE_ERR_CUDA without one
moe_status_t require_sm100();
uint64_t wait_limit_ns();

}  // namespace moe
