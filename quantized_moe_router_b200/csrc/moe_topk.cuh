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

// Lane i < k receives the i-th selected expert (idx) and its weight (w); other lanes get -1/0.
// `l` points to E fp32 logits; `from_l2` selects an L2-only load (data written by other CTAs
// of the same kernel). E <= 1024, 1 <= k <= min(E, 32).
__device__ __forceinline__ void warp_topk_softmax(const float *l, bool from_l2, int E, int k,
                                                  int lane, int &idx, float &w) {
    float v[32];
    uint32_t avail = 0;
#pragma unroll
    for (int m = 0; m < 32; ++m) {
        const int e = lane + 32 * m;
        float x = -INFINITY;
        if (e < E) {
            x = from_l2 ? __ldcg(l + e) : l[e];
            if (x != x) x = -INFINITY;
            avail |= 1u << m;
        }
        v[m] = x;
    }
    int my_i = -1;
    float my_v = -INFINITY;
    for (int r = 0; r < k; ++r) {
        float bv = -INFINITY;
        int be = INT_MAX;
#pragma unroll
        for (int m = 0; m < 32; ++m) {
            const int e = lane + 32 * m;
            if (((avail >> m) & 1u) && (v[m] > bv || (v[m] == bv && e < be))) {
                bv = v[m];
                be = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) avail &= ~(1u << (be >> 5));
        if (lane == r) {
            my_i = be;
            my_v = bv;
        }
    }
    const float v0 = __shfl_sync(0xffffffffu, my_v, 0);
    float ex = 0.f;
    if (lane < k) ex = (v0 == -INFINITY) ? 1.f : expf(my_v - v0);
    float s = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    idx = my_i;
    w = (lane < k) ? ex / s : 0.f;
}

}  // namespace moe
