// Permutation of token slots by expert ("per-expert buffers" of the
// hipfire 0.4.3 benchmarks page, "Read this before comparing columns"
// table): a stable counting sort of the T*k slots s = t*k + j by expert id.
//
//   pass 1: one CTA per 256 slots builds its histogram in shared memory and
//           writes it out; the last CTA to finish (ticket counter) scans the
//           histograms in expert-major order, giving every (CTA, expert)
//           pair its first output position, plus counts and offsets.
//   pass 2: each CTA ranks its slots among equal experts (warp match +
//           per-warp counts, in slot order) and scatters.
// No floating point and no atomics on the outputs: the result is unique.
#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace moeq4 {

constexpr int kPermCh = 256;   // slots per CTA

static inline int perm_blocks(int T, int k) { return (T * k + kPermCh - 1) / kPermCh; }

size_t permute_scratch_bytes(int T, int E, int k)
{
    const size_t nblk = (size_t)perm_blocks(T, k);
    return 256 + 2 * ((nblk * E * sizeof(int32_t) + 255) & ~(size_t)255);
}

__global__ void __launch_bounds__(kPermCh) permute_hist_kernel(const int32_t *__restrict__ ids, int S, int E,
                                                               int32_t *hist, int32_t *base, int32_t *counter,
                                                               int32_t *counts, int32_t *offsets, int *status)
{
    extern __shared__ int32_t s_hist[];   // [E]
    __shared__ int s_last;
    __shared__ int s_part[kPermCh];
    const int nblk = gridDim.x;
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        s_hist[e] = 0;
    __syncthreads();
    const int s = blockIdx.x * kPermCh + threadIdx.x;
    if (s < S) {
        const int e = ids[s];
        if (e >= 0 && e < E)
            atomicAdd(&s_hist[e], 1);
        else
            record_error(status, MOE_ERR_INVALID_ARG, s);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        hist[(size_t)blockIdx.x * E + e] = s_hist[e];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
        s_last = atomicAdd(counter, 1) == nblk - 1;
    __syncthreads();
    if (!s_last)
        return;
    __threadfence();

    // exclusive scan over idx = e * nblk + b of hist[b][e]
    const int N = E * nblk;
    const int per = (N + blockDim.x - 1) / blockDim.x;
    const int i0 = threadIdx.x * per;
    const int i1 = min(N, i0 + per);
    int sum = 0;
    for (int i = i0; i < i1; ++i) {
        const int e = i / nblk, b = i - e * nblk;
        sum += __ldcg(&hist[(size_t)b * E + e]);
    }
    s_part[threadIdx.x] = sum;
    __syncthreads();
    for (int off = 1; off < (int)blockDim.x; off <<= 1) {
        const int v = threadIdx.x >= off ? s_part[threadIdx.x - off] : 0;
        __syncthreads();
        s_part[threadIdx.x] += v;
        __syncthreads();
    }
    int run = s_part[threadIdx.x] - sum;
    for (int i = i0; i < i1; ++i) {
        const int e = i / nblk, b = i - e * nblk;
        base[(size_t)b * E + e] = run;
        if (b == 0)
            offsets[e] = run;
        run += __ldcg(&hist[(size_t)b * E + e]);
    }
    __syncthreads();
    __threadfence_block();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int next = e + 1 < E ? base[e + 1] : S;   // base[0][e+1] lives at index e+1 of row 0
        counts[e] = next - base[e];
    }
    if (threadIdx.x == 0) {
        offsets[E] = S;
        *counter = 0;
    }
}

__global__ void __launch_bounds__(kPermCh) permute_scatter_kernel(const int32_t *__restrict__ ids, int S, int E,
                                                                  const int32_t *__restrict__ base,
                                                                  int32_t *sorted_slot, int32_t *dest_pos)
{
    extern __shared__ int32_t s_wcnt[];   // [8][E]
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int i = threadIdx.x; i < 8 * E; i += blockDim.x)
        s_wcnt[i] = 0;
    __syncthreads();
    const int s = blockIdx.x * kPermCh + threadIdx.x;
    int e = -1;
    if (s < S) {
        e = ids[s];
        if (e < 0 || e >= E)
            e = -1;
    }
    const uint32_t peers = __match_any_sync(0xFFFFFFFFu, e);
    const int rank_w = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && lane == __ffs(peers) - 1)
        s_wcnt[warp * E + e] = __popc(peers);
    __syncthreads();
    if (e >= 0) {
        int rank = rank_w;
        for (int w = 0; w < warp; ++w)
            rank += s_wcnt[w * E + e];
        const int p = base[(size_t)blockIdx.x * E + e] + rank;
        sorted_slot[p] = s;
        dest_pos[s] = p;
    } else if (s < S) {
        dest_pos[s] = -1;
    }
}

cudaError_t launch_permute(const int32_t *ids, int T, int E, int k, int32_t *counts, int32_t *offsets,
                           int32_t *sorted_slot, int32_t *dest_pos, void *scratch, int *status, cudaStream_t st)
{
    const int S = T * k;
    if (S == 0) {
        cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, st);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st);
        return e;
    }
    const int nblk = perm_blocks(T, k);
    uint8_t *sc = (uint8_t *)scratch;
    int32_t *counter = (int32_t *)sc;
    int32_t *hist = (int32_t *)(sc + 256);
    int32_t *base = (int32_t *)(sc + 256 + ((nblk * (size_t)E * sizeof(int32_t) + 255) & ~(size_t)255));
    cudaError_t err = cudaMemsetAsync(counter, 0, sizeof(int32_t), st);
    if (err != cudaSuccess)
        return err;
    permute_hist_kernel<<<nblk, kPermCh, E * sizeof(int32_t), st>>>(ids, S, E, hist, base, counter, counts,
                                                                     offsets, status);
    err = cudaGetLastError();
    if (err != cudaSuccess)
        return err;
    permute_scatter_kernel<<<nblk, kPermCh, 8 * E * sizeof(int32_t), st>>>(ids, S, E, base, sorted_slot,
                                                                          dest_pos);
    return cudaGetLastError();
}

}  // namespace moeq4
