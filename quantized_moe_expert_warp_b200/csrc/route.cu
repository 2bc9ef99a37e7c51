// Top-k routing (the router logits come from the tensor-core GEMM in gemm.cu).
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
#include "ptx.cuh"
#include "topk.cuh"

namespace moeq4 {

// ------------------------------------------------------------------ top-k
// One warp per token (warp_topk in topk.cuh).

// Router logit of (t, e) from split-K partials: slices summed in order,
// then the bias.  Shared by the route and reduce kernels so that both give
// the same bits.
__device__ __forceinline__ float sum_partials(const float *__restrict__ part, int nsplit, size_t TE, size_t idx,
                                              const float *__restrict__ bias, int e)
{
    float acc = part[idx];
    for (int s = 1; s < nsplit; ++s)
        acc += part[(size_t)s * TE + idx];
    return bias ? acc + bias[e] : acc;
}

template <int NPL>
__global__ void __launch_bounds__(128) route_kernel(const float *__restrict__ logits, int T, int E, int k,
                                                    int renorm, int32_t *ids, float *w,
                                                    const float *__restrict__ part, int nsplit,
                                                    const float *__restrict__ bias, float *logits_out)
{
    pdl_wait();
    pdl_allow_successor();
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    if (warp >= T)
        return;
    float v[NPL];
    if (part) {
        // the same order as sum_partials: slice 0, 1, ..., then the bias;
        // all of a slice's loads are issued together
        const size_t TE = (size_t)T * E;
        const float *row = part + (size_t)warp * E;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = i * 32 + lane;
            v[i] = e < E ? row[e] : 0.f;
        }
        // slices 1, 2, ... in groups (four while the values fit in registers):
        // a group's loads are issued together, then added in slice order
        constexpr int G = NPL <= 8 ? 4 : 1;
        for (int sl = 1; sl < nsplit; sl += G) {
            float g[G][NPL];
#pragma unroll
            for (int q = 0; q < G; ++q) {
                const float *r = row + (size_t)(sl + q) * TE;
#pragma unroll
                for (int i = 0; i < NPL; ++i) {
                    const int e = i * 32 + lane;
                    g[q][i] = sl + q < nsplit && e < E ? r[e] : 0.f;
                }
            }
#pragma unroll
            for (int q = 0; q < G; ++q)
#pragma unroll
                for (int i = 0; i < NPL; ++i)
                    if (sl + q < nsplit && i * 32 + lane < E)
                        v[i] += g[q][i];
        }
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = i * 32 + lane;
            if (e < E) {
                if (bias)
                    v[i] += bias[e];
                if (logits_out)
                    logits_out[(size_t)warp * E + e] = v[i];
            } else {
                v[i] = -CUDART_INF_F;
            }
        }
    } else {
        const float *L = logits + (size_t)warp * E;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = i * 32 + lane;
            v[i] = e < E ? L[e] : -CUDART_INF_F;
        }
    }
    float top, my_val;
    int my_id;
    warp_topk<NPL>(v, E, k, lane, my_val, my_id, top);
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
        // a position left unfilled (NaN logits) gets id -1 and weight 0; the
        // permutation reports such ids as out of range
        const bool filled = my_id != 0x7FFFFFFF;
        ids[(size_t)warp * k + lane] = filled ? my_id : -1;
        w[(size_t)warp * k + lane] = filled ? ex / z : 0.f;
    }
}

cudaError_t launch_route(const float *logits, int T, int E, int k, int renorm, int32_t *ids, float *w,
                         cudaStream_t st, const float *part, int nsplit, const float *bias, float *logits_out)
{
    if (T == 0)
        return cudaSuccess;
    const int blocks = (T + 3) / 4;   // four tokens (warps) per block: more SMs share the partial reads
    const int npl = (E + 31) / 32;
#define ROUTE_ARGS logits, T, E, k, renorm, ids, w, part, nsplit, bias, logits_out
    if (npl <= 1)
        return launch_pdl(route_kernel<1>, blocks, 128, 0, st, ROUTE_ARGS);
    if (npl <= 2)
        return launch_pdl(route_kernel<2>, blocks, 128, 0, st, ROUTE_ARGS);
    if (npl <= 4)
        return launch_pdl(route_kernel<4>, blocks, 128, 0, st, ROUTE_ARGS);
    if (npl <= 8)
        return launch_pdl(route_kernel<8>, blocks, 128, 0, st, ROUTE_ARGS);
    if (npl <= 16)
        return launch_pdl(route_kernel<16>, blocks, 128, 0, st, ROUTE_ARGS);
    return launch_pdl(route_kernel<32>, blocks, 128, 0, st, ROUTE_ARGS);
#undef ROUTE_ARGS
}

__global__ void __launch_bounds__(256) router_reduce_kernel(const float *__restrict__ part, int nsplit, int T, int E,
                                                            const float *__restrict__ bias, float *logits)
{
    pdl_wait();
    pdl_allow_successor();
    const size_t TE = (size_t)T * E;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < TE; i += (size_t)gridDim.x * blockDim.x)
        logits[i] = sum_partials(part, nsplit, TE, i, bias, (int)(i % E));
}

cudaError_t launch_router_reduce(const float *part, int nsplit, int T, int E, const float *bias, float *logits,
                                 cudaStream_t st)
{
    const size_t TE = (size_t)T * E;
    if (TE == 0)
        return cudaSuccess;
    const int blocks = (int)((TE + 255) / 256 < 4096 ? (TE + 255) / 256 : 4096);
    return launch_pdl(router_reduce_kernel, blocks, 256, 0, st, part, nsplit, T, E, bias, logits);
}

}  // namespace moeq4
