// Warp-level top-k selection shared by the route kernel and the fused decode kernel.
//
// One warp holds one token's E logits, lane l the logits l, l + 32, ...
// (v[i] is logit i * 32 + lane).  Each of the k rounds takes the warp's
// maximum with two warp reductions (redux.sync): the largest order key of
// the lanes' own best remaining logits, then the smallest expert id among
// the lanes that hold that key.  Ties therefore go to the lower id, -0 and
// +0 are equal, and NaN logits are never chosen.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <math_constants.h>

namespace moeq4 {

// Order key of a logit: larger logits give larger unsigned keys; NaN gives 0.
__device__ __forceinline__ uint32_t order_key(float v)
{
    if (v != v)
        return 0u;
    const uint32_t b = __float_as_uint(v == 0.f ? 0.f : v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Lane j < k gets the j-th largest logit (val) and its expert id (id;
// 0x7FFFFFFF and val = -inf where every remaining logit is NaN); every lane
// gets the largest logit (top).
template <int NPL>
__device__ __forceinline__ void warp_topk(const float (&v)[NPL], int E, int k, int lane, float &my_val, int &my_id,
                                          float &top)
{
    uint32_t key[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i)
        key[i] = i * 32 + lane < E ? order_key(v[i]) : 0u;
    top = 0.f;
    my_val = -CUDART_INF_F;
    my_id = 0x7FFFFFFF;
    for (int j = 0; j < k; ++j) {
        // this lane's best remaining logit (the lowest id among equal keys)
        uint32_t bk = 0u;
        int bi = 0;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            if (key[i] > bk) {
                bk = key[i];
                bi = i;
            }
        const uint32_t wk = __reduce_max_sync(0xFFFFFFFFu, bk);
        const int bid = (int)__reduce_min_sync(0xFFFFFFFFu, (wk != 0u && bk == wk) ? (uint32_t)(bi * 32 + lane)
                                                                                   : 0x7FFFFFFFu);
        float val = -CUDART_INF_F;   // an unfilled position adds nothing to the softmax sums
        if (bid != 0x7FFFFFFF) {     // warp-uniform
            float mine = 0.f;
#pragma unroll
            for (int i = 0; i < NPL; ++i)
                if (i == (bid >> 5)) {
                    mine = v[i];
                    if ((bid & 31) == lane)
                        key[i] = 0u;   // taken
                }
            val = __shfl_sync(0xFFFFFFFFu, mine, bid & 31);
        }
        if (j == 0)
            top = val;
        if (lane == j) {
            my_val = val;
            my_id = bid;
        }
    }
}

}  // namespace moeq4
