// Router logits and top-k routing.
//
// The pages run Qwen3-family MoE models (hipfire 0.4.3 benchmarks,
// "Qwen3.6-35B-A3B prefill on the R9700"; hipEngine post, "Benchmarks vs
// llama.cpp") but print no routing rule.  Reading used here: softmax over
// the router logits, the k largest kept (ties to the lower expert id, in
// descending order), weights renormalised over the kept k.
#include <cstdint>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kernels.h"

namespace moeq4 {

// ------------------------------------------------------------ router logits
// logits[t, e] = sum_h x[t, h] * Wr[e, h] (+ bias[e]) in fp32; row E of the
// tile (when gate_w is given) produces the shared expert's gate logit.
constexpr int kRT = 64;   // tokens per CTA
constexpr int kRR = 64;   // router rows per CTA
constexpr int kRK = 32;   // K per smem stage

__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t *__restrict__ x, int T, int H,
                                                            const float *__restrict__ wr,
                                                            const float *__restrict__ bias, int E,
                                                            const float *__restrict__ gate_w, float *logits,
                                                            float *gate_logit)
{
    __shared__ float xs[kRK][kRT + 4];
    __shared__ float ws[kRK][kRR + 4];
    const int R = E + (gate_w ? 1 : 0);
    const int t0 = blockIdx.x * kRT;
    const int r0 = blockIdx.y * kRR;
    const int tid = threadIdx.x;
    const int ty = tid / 16, tx = tid % 16;
    float acc[4][4] = {};

    const int lrow = tid / 4;          // 0..63
    const int lk = (tid % 4) * 8;      // 0, 8, 16, 24
    const int lt = t0 + lrow;
    const int lr = r0 + lrow;
    const float *wrow = lr < E ? wr + (size_t)lr * H : (lr == E && gate_w ? gate_w : nullptr);

    for (int kb = 0; kb < H; kb += kRK) {
        if (lt < T) {
            const uint4 v = *(const uint4 *)(x + (size_t)lt * H + kb + lk);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xs[lk + 2 * i][lrow] = __uint_as_float(w4[i] << 16);
                xs[lk + 2 * i + 1][lrow] = __uint_as_float(w4[i] & 0xFFFF0000u);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                xs[lk + i][lrow] = 0.f;
        }
        if (wrow) {
            const float4 a = *(const float4 *)(wrow + kb + lk);
            const float4 b = *(const float4 *)(wrow + kb + lk + 4);
            ws[lk + 0][lrow] = a.x; ws[lk + 1][lrow] = a.y; ws[lk + 2][lrow] = a.z; ws[lk + 3][lrow] = a.w;
            ws[lk + 4][lrow] = b.x; ws[lk + 5][lrow] = b.y; ws[lk + 6][lrow] = b.z; ws[lk + 7][lrow] = b.w;
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                ws[lk + i][lrow] = 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < kRK; ++kk) {
            const float4 xa = *(const float4 *)&xs[kk][ty * 4];
            const float4 wa = *(const float4 *)&ws[kk][tx * 4];
            const float xv[4] = {xa.x, xa.y, xa.z, xa.w};
            const float wv[4] = {wa.x, wa.y, wa.z, wa.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    acc[i][j] = fmaf(xv[i], wv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + ty * 4 + i;
        if (t >= T)
            continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = r0 + tx * 4 + j;
            if (r < E)
                logits[(size_t)t * E + r] = acc[i][j] + (bias ? bias[r] : 0.f);
            else if (r == E && r < R)
                gate_logit[t] = acc[i][j];
        }
    }
}

cudaError_t launch_router_logits(const uint16_t *x, int T, int H, const float *wr, const float *bias, int E,
                                 const float *gate_w, float *logits, float *gate_logit, cudaStream_t st)
{
    if (T == 0)
        return cudaSuccess;
    const int R = E + (gate_w ? 1 : 0);
    dim3 grid((T + kRT - 1) / kRT, (R + kRR - 1) / kRR);
    router_logits_kernel<<<grid, 256, 0, st>>>(x, T, H, wr, bias, E, gate_w, logits, gate_logit);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ top-k
// One warp per token; lane l holds logits l, l+32, ... in registers.

__device__ __forceinline__ bool better(float v, int id, float bv, int bid)
{
    return v > bv || (v == bv && id < bid);
}

template <int NPL>
__global__ void __launch_bounds__(256) route_kernel(const float *__restrict__ logits, int T, int E, int k,
                                                    int renorm, int32_t *ids, float *w)
{
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    if (warp >= T)
        return;
    const float *L = logits + (size_t)warp * E;
    float v[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = i * 32 + lane;
        v[i] = e < E ? L[e] : -CUDART_INF_F;
    }
    uint32_t taken = 0;
    float top = 0.f, my_val = 0.f;
    int my_id = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -CUDART_INF_F;
        int bid = 0x7FFFFFFF;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = i * 32 + lane;
            if (e < E && !((taken >> i) & 1u) && better(v[i], e, bv, bid)) {
                bv = v[i];
                bid = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
            const int oid = __shfl_xor_sync(0xFFFFFFFFu, bid, off);
            if (better(ov, oid, bv, bid)) {
                bv = ov;
                bid = oid;
            }
        }
        if ((bid & 31) == lane)
            taken |= 1u << (bid >> 5);
        if (j == 0)
            top = bv;
        if (lane == j) {
            my_val = bv;
            my_id = bid;
        }
    }
    const float ex = lane < k ? expf(my_val - top) : 0.f;
    float z;
    if (renorm) {
        // sum of the kept k in j order
        z = 0.f;
        for (int j = 0; j < k; ++j)
            z += __shfl_sync(0xFFFFFFFFu, ex, j);
    } else {
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            if (i * 32 + lane < E)
                part += expf(v[i] - top);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            part += __shfl_xor_sync(0xFFFFFFFFu, part, off);
        z = part;
    }
    if (lane < k) {
        ids[(size_t)warp * k + lane] = my_id;
        w[(size_t)warp * k + lane] = ex / z;
    }
}

cudaError_t launch_route(const float *logits, int T, int E, int k, int renorm, int32_t *ids, float *w,
                         cudaStream_t st)
{
    if (T == 0)
        return cudaSuccess;
    const int blocks = (T + 7) / 8;
    const int npl = (E + 31) / 32;
    if (npl <= 1)
        route_kernel<1><<<blocks, 256, 0, st>>>(logits, T, E, k, renorm, ids, w);
    else if (npl <= 2)
        route_kernel<2><<<blocks, 256, 0, st>>>(logits, T, E, k, renorm, ids, w);
    else if (npl <= 4)
        route_kernel<4><<<blocks, 256, 0, st>>>(logits, T, E, k, renorm, ids, w);
    else if (npl <= 8)
        route_kernel<8><<<blocks, 256, 0, st>>>(logits, T, E, k, renorm, ids, w);
    else if (npl <= 16)
        route_kernel<16><<<blocks, 256, 0, st>>>(logits, T, E, k, renorm, ids, w);
    else
        route_kernel<32><<<blocks, 256, 0, st>>>(logits, T, E, k, renorm, ids, w);
    return cudaGetLastError();
}

}  // namespace moeq4
