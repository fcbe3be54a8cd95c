// moe_topk.cuh -- warp-cooperative top-k with softmax renormalisation.
//
// Selection order: larger logit first; equal logits -> lower expert index (the tie rule of
// the block's routing step); NaN logits rank as -inf. Weights: w_i = exp(l_i - l_max) /
// sum_{j in top-k} exp(l_j - l_max), i.e. the softmax restricted to the selected experts
// (the renormalised routing weights of the MoE block used on the pages "--moe-direct-io"
// and "Qwen-tin" with 512 experts and top-10 routing).
#pragma once
#include <cfloat>
#include <climits>
#include "moe_internal.cuh"

namespace moe {

// monotone map of a non-NaN float to an unsigned key (larger float -> larger key)
__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Largest key of a lane's M keys and its position, equal keys -> the lower position (the lower
// expert index); written with selects (a divergent branch per key costs far more).
template <int M>
__device__ __forceinline__ void lane_max_key(const uint32_t (&key)[M], uint32_t &bk, int &bm) {
    bk = key[0];
    bm = 0;
#pragma unroll
    for (int m = 1; m < M; ++m) {
        const bool gt = key[m] > bk;
        bk = gt ? key[m] : bk;
        bm = gt ? m : bm;
    }
}

// Lane i < k receives the i-th selected expert (idx) and its weight (w); other lanes get -1/0.
// `l` points to E fp32 logits; `from_l2` selects an L2-only load (data written by other CTAs
// of the same kernel). E <= 32 M, 1 <= k <= min(E, 32).
// Each round takes the warp-wide maximum key and then the lowest index holding it (two redux
// instructions); only the winning lane rescans its M keys.
template <int M>
__device__ __forceinline__ void warp_topk_softmax_m(const float *l, bool from_l2, int E, int k, int lane, int &idx,
                                                    float &w) {
    // lane holds logits lane + 32 m (m < M) as order keys; 0 = taken / absent
    uint32_t key[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
        const int e = lane + 32 * m;
        uint32_t kk = 0;
        if (e < E) {
            float x = from_l2 ? __ldcg(l + e) : l[e];
            if (x != x) x = -INFINITY;
            kk = order_key(x);   // >= 0x007FFFFF for -inf, so never 0
        }
        key[m] = kk;
    }
    uint32_t bk;
    int bm;
    lane_max_key<M>(key, bk, bm);
    int my_i = -1;
    uint32_t my_k = 0;
    for (int r = 0; r < k; ++r) {
        const uint32_t mx = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t cand = (bk == mx) ? (uint32_t)(lane + 32 * bm) : 0xFFFFFFFFu;
        const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
        if (lane == r) {
            my_i = (int)win;
            my_k = mx;
        }
        // the winning lane drops its entry and rescans (selects, no branch per key)
        const bool mine = (int)(win & 31u) == lane;
#pragma unroll
        for (int m = 0; m < M; ++m) key[m] = (mine && m == bm) ? 0u : key[m];
        if (mine) lane_max_key<M>(key, bk, bm);
    }
    const float my_v = (lane < k) ? key_value(my_k) : -INFINITY;
    const float v0 = __shfl_sync(0xffffffffu, my_v, 0);
    float ex = 0.f;
    if (lane < k) ex = (v0 == -INFINITY) ? 1.f : expf(my_v - v0);
    float s = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    idx = my_i;
    w = (lane < k) ? ex / s : 0.f;
}

// E <= 1024: the register list sized to the expert count
__device__ __forceinline__ void warp_topk_softmax(const float *l, bool from_l2, int E, int k, int lane, int &idx,
                                                  float &w) {
    if (E <= 64) warp_topk_softmax_m<2>(l, from_l2, E, k, lane, idx, w);
    else if (E <= 256) warp_topk_softmax_m<8>(l, from_l2, E, k, lane, idx, w);
    else if (E <= 512) warp_topk_softmax_m<16>(l, from_l2, E, k, lane, idx, w);
    else warp_topk_softmax_m<32>(l, from_l2, E, k, lane, idx, w);
}

}  // namespace moe
