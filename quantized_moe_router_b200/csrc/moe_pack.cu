// moe_pack.cu -- canonical expert tensors -> the packed tile layout of moe_internal.cuh.
//
// A pure byte/bit permutation (no value is rounded): each thread builds one lane's share of one
// 16x64 tile -- its 16 lo-plane bytes, its hi-plane bytes and (for t == 0) its scale/zero entry --
// and stores it at the tile's place (gate/up) or scatters it over the four quarters of its
// super-tile (down).
#include "moe_internal.cuh"

namespace moe {
namespace {

struct PackSrc {
    const uint8_t *codes[3];
    const uint16_t *scale[3];
    const uint16_t *zero[3];
};

// code (row, col) of a canonical matrix with `cols` columns and `bits`-bit codes
__device__ __forceinline__ uint32_t canon_code(const uint8_t *codes, int cols, int bits, int row, int col) {
    const uint8_t *blk = codes + (size_t)row * ((size_t)cols * bits / 8) + (size_t)(col / kGroup) * 8 * bits;
    const uint32_t bit = (uint32_t)(col % kGroup) * bits;
    const uint32_t byte = bit >> 3, sh = bit & 7;
    uint32_t v = blk[byte];
    if (sh + bits > 8) v |= (uint32_t)blk[byte + 1] << 8;
    return (v >> sh) & ((1u << bits) - 1u);
}

template <int BITS>
__global__ void pack_expert_kernel(PackSrc src, int H, int I, uint8_t *dst, long long ntile_lanes,
                                   PackedHeader hdr, int e, PackedExpert entry, uint8_t *packed) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        if (e == 0) *reinterpret_cast<PackedHeader *>(packed) = hdr;
        reinterpret_cast<PackedExpert *>(packed + sizeof(PackedHeader))[e] = entry;
    }
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= ntile_lanes) return;
    const long long tile = gid >> 5;
    const int lane = (int)(gid & 31), g = lane >> 2, t = lane & 3;
    const long long ngu = (long long)gu_tiles(H, I);
    int mA, mB, rowA, rowB, cols, kg;
    if (tile < ngu) {
        const int G = H / kGroup;
        const int rb = (int)(tile / G);
        kg = (int)(tile % G);
        mA = 0; mB = 1; rowA = rb * 8 + g; rowB = rb * 8 + g; cols = H;
    } else {
        const int GI = I / kGroup;
        const long long dt = tile - ngu;
        const int rb = (int)(dt / GI);
        kg = (int)(dt % GI);
        mA = 2; mB = 2; rowA = rb * 16 + g; rowB = rb * 16 + g + 8; cols = I;
    }
    uint32_t lo[4], hi8[4], hi6[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int kb = kg * kGroup + 16 * t + 4 * j;
        // operand elements a0..a7 of MMA j (rows g / g+8, group columns kb..kb+3)
        uint32_t a[8];
        a[0] = canon_code(src.codes[mA], cols, BITS, rowA, kb + 0);
        a[1] = canon_code(src.codes[mA], cols, BITS, rowA, kb + 1);
        a[2] = canon_code(src.codes[mB], cols, BITS, rowB, kb + 0);
        a[3] = canon_code(src.codes[mB], cols, BITS, rowB, kb + 1);
        a[4] = canon_code(src.codes[mA], cols, BITS, rowA, kb + 2);
        a[5] = canon_code(src.codes[mA], cols, BITS, rowA, kb + 3);
        a[6] = canon_code(src.codes[mB], cols, BITS, rowB, kb + 2);
        a[7] = canon_code(src.codes[mB], cols, BITS, rowB, kb + 3);
        uint32_t wl = 0, wh = 0;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            wl |= (a[2 * r] & 15u) << (4 * r);
            wl |= (a[2 * r + 1] & 15u) << (16 + 4 * r);
            wh |= ((a[2 * r] >> 4) & 15u) << (4 * r);
            wh |= ((a[2 * r + 1] >> 4) & 15u) << (16 + 4 * r);
            const int s = 4 * (j & 1) + r;  // 6-bit hi: pair s of word j/2
            hi6[j >> 1] |= ((a[2 * r] >> 4) & 3u) << (2 * s);
            hi6[j >> 1] |= ((a[2 * r + 1] >> 4) & 3u) << (16 + 2 * s);
        }
        lo[j] = wl;
        hi8[j] = wh;
    }
    const int GA = cols / kGroup;
    uint2 sz = make_uint2(0u, 0u);
    if (t == 0) {
        const uint32_t sA = src.scale[mA][(size_t)rowA * GA + kg], zA = src.zero[mA][(size_t)rowA * GA + kg];
        const uint32_t sB = src.scale[mB][(size_t)rowB * GA + kg], zB = src.zero[mB][(size_t)rowB * GA + kg];
        sz = make_uint2(sA | (zA << 16), sB | (zB << 16));
    }
    if (tile < ngu) {
        // row blocks 2i and 2i + 1 (16 intermediate rows) interleaved along K: tile (rb, kg) at
        // ((rb / 2) * KG + kg) * 2 + rb % 2
        const int KG = H / kGroup, rb = (int)(tile / KG);
        const long long pos = ((long long)(rb >> 1) * KG + kg) * 2 + (rb & 1);
        uint8_t *tp = dst + pos * tile_bytes(BITS);
        *reinterpret_cast<uint4 *>(tp + 16 * lane) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        if (BITS == 8) *reinterpret_cast<uint4 *>(tp + kLoBytes + 16 * lane) = make_uint4(hi8[0], hi8[1], hi8[2], hi8[3]);
        if (BITS == 6) *reinterpret_cast<uint2 *>(tp + kLoBytes + 8 * lane) = make_uint2(hi6[0], hi6[1]);
        if (t == 0) *reinterpret_cast<uint2 *>(tp + kLoBytes + hi_bytes(BITS) + 8 * g) = sz;
    } else {
        // word j of this lane (g, t) is word (r, lane 4g + j) of quarter t of super-tile st
        const int rb = rowA / 16, st = rb >> 2, r = rb & 3;
        uint8_t *blk = dst + (size_t)ngu * tile_bytes(BITS) + (size_t)kg * d_block_bytes(H, BITS);
        uint8_t *qp = blk + d_quarter_offset(H, BITS, t) + (size_t)st * d_quarter_bytes(BITS);
        *reinterpret_cast<uint4 *>(qp + r * 128 + 16 * g) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        if (BITS == 8) *reinterpret_cast<uint4 *>(qp + kLoBytes + r * 128 + 16 * g) = make_uint4(hi8[0], hi8[1], hi8[2], hi8[3]);
        if (BITS == 6) {
            // MMA j's two bytes of hi word j/2 (bits 8(j%2).. and 16+8(j%2)..) as one half-word
            uint32_t h[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t w = hi6[j >> 1] >> (8 * (j & 1));
                h[j] = (w & 0xFFu) | ((w >> 8) & 0xFF00u);
            }
            *reinterpret_cast<uint2 *>(qp + kLoBytes + r * 64 + 8 * g) = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
        }
        if (t == 0) *reinterpret_cast<uint2 *>(blk + (size_t)st * 256 + r * 64 + 8 * g) = sz;
    }
}

}  // namespace

size_t packed_layer_bytes(int E, int H, int I, const int32_t *bits) {
    size_t o = packed_data_start(E);
    for (int e = 0; e < E; ++e) o = align_up(o + expert_bytes(H, I, bits[e]), 256);
    return o;
}

moe_status_t launch_pack(const moe_expert_src_t *src, int E, int H, int I, void *packed, cudaStream_t st) {
    PackedHeader hdr = {};
    hdr.magic = kPackedMagic;
    hdr.version = kPackedVersion;
    hdr.E = E; hdr.H = H; hdr.I = I;
    size_t off = packed_data_start(E);
    uint8_t *p8 = static_cast<uint8_t *>(packed);
    for (int e = 0; e < E; ++e) {
        const int bits = src[e].bits;
        PackSrc ps;
        for (int m = 0; m < 3; ++m) {
            ps.codes[m] = static_cast<const uint8_t *>(src[e].codes[m]);
            ps.scale[m] = src[e].scale[m];
            ps.zero[m] = src[e].zero[m];
        }
        PackedExpert entry = {off, bits, 0};
        const long long lanes = (long long)(gu_tiles(H, I) + d_tiles(H, I)) * 32;
        const int threads = 256;
        const unsigned blocks = (unsigned)((lanes + threads - 1) / threads);
        if (bits == 4)
            pack_expert_kernel<4><<<blocks, threads, 0, st>>>(ps, H, I, p8 + off, lanes, hdr, e, entry, p8);
        else if (bits == 6)
            pack_expert_kernel<6><<<blocks, threads, 0, st>>>(ps, H, I, p8 + off, lanes, hdr, e, entry, p8);
        else
            pack_expert_kernel<8><<<blocks, threads, 0, st>>>(ps, H, I, p8 + off, lanes, hdr, e, entry, p8);
        if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
        off = align_up(off + expert_bytes(H, I, bits), 256);
    }
    return MOE_OK;
}

}  // namespace moe
