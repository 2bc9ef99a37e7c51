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

// The logit of an order key (not 0).
__device__ __forceinline__ float key_value(uint32_t key)
{
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Lane j < k gets the j-th largest logit (my_val; a -0 logit as +0) and its
// expert id (my_id; 0x7FFFFFFF and my_val = -inf where every remaining
// logit is NaN); every lane gets the largest logit (top).  The owner lane
// marks its chosen logit in a bit mask, and the value is recovered from the
// winning key.
template <int NPL>
__device__ __forceinline__ void warp_topk(const float (&v)[NPL], int E, int k, int lane, float &my_val, int &my_id,
                                          float &top)
{
    // order keys once; a chosen logit is masked through the taken bits (no
    // write into the key array, which would need a dynamic index)
    uint32_t key[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i)
        key[i] = i * 32 + lane < E ? order_key(v[i]) : 0u;
    uint32_t taken = 0u;   // bit i: logit i * 32 + lane already chosen
    top = 0.f;
    my_val = -CUDART_INF_F;
    my_id = 0x7FFFFFFF;
    for (int j = 0; j < k; ++j) {
        // this lane's best remaining logit (the lowest id among equal keys)
        uint32_t bk = 0u;
        int bi = 0;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const uint32_t ki = (taken >> i) & 1u ? 0u : key[i];
            if (ki > bk) {
                bk = ki;
                bi = i;
            }
        }
        const uint32_t wk = __reduce_max_sync(0xFFFFFFFFu, bk);
        const int bid = (int)__reduce_min_sync(0xFFFFFFFFu, (wk != 0u && bk == wk) ? (uint32_t)(bi * 32 + lane)
                                                                                   : 0x7FFFFFFFu);
        // the chosen logit is the key's inverse (a -0 logit comes back as +0, which
        // changes no softmax term); an unfilled position adds nothing to the sums
        float val = -CUDART_INF_F;
        if (bid != 0x7FFFFFFF) {   // warp-uniform
            val = key_value(wk);
            if ((bid & 31) == lane)
                taken |= 1u << (bid >> 5);
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
