// Weighted combine: y[t] = sum_j w[t,j] Y[dest_pos[t k + j]] + sigmoid(g_t) S[t].
//
// The pages state no combine rule; reading: the standard top-k mixture of
// the routed experts' outputs plus the sigmoid-gated shared expert of the
// Qwen3-Next-style layers run on the hipfire 0.4.3 benchmarks page.
// Each thread owns 8 consecutive features of a token and reads them with
// 16-byte loads (coalesced across the warp); fp32 sums in j order, the
// shared expert last.  For k <= 8 and H <= 2048 (the common shapes) the
// kernel is persistent: a thread takes the same features of tokens t,
// t + G, ... and loads the next token's rows before it sums the current
// ones, so that every thread keeps two tokens' loads in flight; other shapes
// take one CTA per token (or per few tokens) and batches of 8 rows.  Both
// forms add in the same order, so they give the same bits.
#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace moeq4 {

__device__ __forceinline__ void add8(float (&acc)[8], const uint4 v, float w)
{
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(w, __uint_as_float(u[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = fmaf(w, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
    }
}

__global__ void __launch_bounds__(256) combine_kernel(const uint16_t *__restrict__ y_perm,
                                                      const int32_t *__restrict__ dest_pos,
                                                      const float *__restrict__ w,
                                                      const uint16_t *__restrict__ shared_out,
                                                      const float *__restrict__ gate_logit, int T, int H, int k,
                                                      uint16_t *__restrict__ y)
{
    pdl_wait();
    pdl_allow_successor();
    const int chunks = H / 8;
    const int per_cta_tokens = blockDim.x / chunks > 0 ? blockDim.x / chunks : 1;
    if ((int)threadIdx.x / chunks >= per_cta_tokens)
        return;
    const int t = blockIdx.x * per_cta_tokens + threadIdx.x / chunks;
    if (t >= T)
        return;
    const int S = T * k;
    const int32_t *dp = dest_pos + (size_t)t * k;
    const float *wt = w + (size_t)t * k;
    // the shared expert's gate, once per token
    const float g = shared_out && gate_logit ? 1.0f / (1.0f + expf(-gate_logit[t])) : 1.0f;
    for (int c = threadIdx.x % chunks; c < chunks; c += blockDim.x) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        // the shared expert's row is loaded with the first batch, added last
        const uint4 sv = shared_out ? __ldcs((const uint4 *)(shared_out + (size_t)t * H + c * 8)) : make_uint4(0, 0, 0, 0);
        // batches of 8 rows: all loads of a batch are in flight together
        for (int j0 = 0; j0 < k; j0 += 8) {
            uint4 v[8];
            float wj[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int p = j0 + j < k ? dp[j0 + j] : -1;
                const bool ok = p >= 0 && p < S;
                wj[j] = ok ? wt[j0 + j] : 0.f;
                // each row is read once: streaming loads keep it out of the way in L1 and L2
                v[j] = ok ? __ldcs((const uint4 *)(y_perm + (size_t)p * H + c * 8)) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j0 + j < k)
                    add8(acc, v[j], wj[j]);
        }
        if (shared_out)
            add8(acc, sv, g);
        uint4 o;
        uint32_t *ou = &o.x;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t d;
            asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(acc[2 * i + 1]), "f"(acc[2 * i]));
            ou[i] = d;
        }
        *(uint4 *)(y + (size_t)t * H + c * 8) = o;
    }
}

// Persistent form for k <= 8 and H / 8 <= blockDim.x: thread (token slot,
// chunk c) of CTA b takes tokens t = (b + G i) per + slot.
struct CombineRows {
    uint4 v[8];
    float w[8];
    uint4 sv;
    float g;
};

__device__ __forceinline__ void combine_load(CombineRows &r, const uint16_t *__restrict__ y_perm,
                                             const int32_t *__restrict__ dest_pos, const float *__restrict__ w,
                                             const uint16_t *__restrict__ shared_out,
                                             const float *__restrict__ gate_logit, int t, int c, int H, int k, int S)
{
    const int32_t *dp = dest_pos + (size_t)t * k;
    const float *wt = w + (size_t)t * k;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int p = j < k ? dp[j] : -1;
        const bool ok = p >= 0 && p < S;
        r.w[j] = ok ? wt[j] : 0.f;
        r.v[j] = ok ? __ldcs((const uint4 *)(y_perm + (size_t)p * H + c * 8)) : make_uint4(0, 0, 0, 0);
    }
    r.sv = shared_out ? __ldcs((const uint4 *)(shared_out + (size_t)t * H + c * 8)) : make_uint4(0, 0, 0, 0);
    r.g = shared_out && gate_logit ? gate_logit[t] : 0.f;
}

__global__ void __launch_bounds__(256) combine_persistent_kernel(const uint16_t *__restrict__ y_perm,
                                                                 const int32_t *__restrict__ dest_pos,
                                                                 const float *__restrict__ w,
                                                                 const uint16_t *__restrict__ shared_out,
                                                                 const float *__restrict__ gate_logit, int T, int H,
                                                                 int k, uint16_t *__restrict__ y)
{
    pdl_wait();
    pdl_allow_successor();
    const int chunks = H / 8;
    const int per = blockDim.x / chunks;
    const int slot = (int)threadIdx.x / chunks, c = (int)threadIdx.x % chunks;
    if (slot >= per)
        return;
    const int S = T * k;
    const int step = gridDim.x * per;
    int t = blockIdx.x * per + slot;
    if (t >= T)
        return;
    CombineRows cur, nxt;
    combine_load(cur, y_perm, dest_pos, w, shared_out, gate_logit, t, c, H, k, S);
    for (;;) {
        const int tn = t + step;
        if (tn < T)
            combine_load(nxt, y_perm, dest_pos, w, shared_out, gate_logit, tn, c, H, k, S);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j < k)
                add8(acc, cur.v[j], cur.w[j]);
        if (shared_out)
            add8(acc, cur.sv, gate_logit ? 1.0f / (1.0f + expf(-cur.g)) : 1.0f);
        uint4 o;
        uint32_t *ou = &o.x;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t d;
            asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(acc[2 * i + 1]), "f"(acc[2 * i]));
            ou[i] = d;
        }
        *(uint4 *)(y + (size_t)t * H + c * 8) = o;
        if (tn >= T)
            break;
        cur = nxt;
        t = tn;
    }
}

cudaError_t launch_combine(const uint16_t *y_perm, const int32_t *dest_pos, const float *w, const uint16_t *shared_out,
                           const float *gate_logit, int T, int H, int k, uint16_t *y, int num_sms, cudaStream_t st)
{
    if (T == 0)
        return cudaSuccess;
    const int chunks = H / 8;
    const int threads = 256;
    const int per = threads / chunks > 0 ? threads / chunks : 1;
    if (k <= 8 && chunks <= threads) {
        // two CTAs per SM stay resident (about 100 registers a thread)
        const int want = 2 * (num_sms > 0 ? num_sms : 1);
        const int need = (T + per - 1) / per;
        return launch_pdl(combine_persistent_kernel, need < want ? need : want, threads, 0, st, y_perm, dest_pos, w,
                          shared_out, gate_logit, T, H, k, y);
    }
    return launch_pdl(combine_kernel, (T + per - 1) / per, threads, 0, st, y_perm, dest_pos, w, shared_out, gate_logit,
                      T, H, k, y);
}

}  // namespace moeq4
