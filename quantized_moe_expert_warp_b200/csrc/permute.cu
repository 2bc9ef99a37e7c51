// Permutation of token slots by expert ("per-expert buffers" of the
// hipfire 0.4.3 benchmarks page, "Read this before comparing columns"
// table): a stable counting sort of the T*k slots s = t*k + j by expert id.
//
//   pass 1: the slots are cut into at most 32 contiguous chunks; one CTA per
//           chunk builds the chunk's expert histogram in shared memory.
//   pass 2: each CTA reads all chunk histograms (at most 32 x E counts),
//           derives every expert's offset and its own chunk's first position
//           per expert, then ranks its slots in slot order (warp match plus
//           per-warp counts) and scatters.  CTA 0 writes counts and offsets.
// No floating point and no atomics on the outputs: the result is unique.
#include <cstdint>
#include <mutex>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace moeq4 {

constexpr int kPermThreads = 1024;
constexpr int kPermMaxChunks = 32;

static inline int perm_chunk(int S)
{
    const int per = (S + kPermMaxChunks - 1) / kPermMaxChunks;
    return ((per + kPermThreads - 1) / kPermThreads) * kPermThreads;
}

static inline int perm_blocks(int S) { return S == 0 ? 0 : (S + perm_chunk(S) - 1) / perm_chunk(S); }

size_t permute_scratch_bytes(int T, int E, int k)
{
    return ((size_t)kPermMaxChunks * E * sizeof(int32_t) + 255) & ~(size_t)255;
}

__global__ void __launch_bounds__(kPermThreads) permute_hist_kernel(const int32_t *__restrict__ ids, int S, int E,
                                                                    int chunk, int32_t *hist, int *status)
{
    pdl_wait();
    pdl_allow_successor();
    extern __shared__ int32_t s_hist[];   // [E]
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        s_hist[e] = 0;
    __syncthreads();
    const int s1 = min(S, (blockIdx.x + 1) * chunk);
    for (int s = blockIdx.x * chunk + threadIdx.x; s < s1; s += blockDim.x) {
        const int e = ids[s];
        if (e >= 0 && e < E)
            atomicAdd(&s_hist[e], 1);
        else
            record_error(status, MOE_ERR_INVALID_ARG, s);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        hist[(size_t)blockIdx.x * E + e] = s_hist[e];
}

// Ranks and scatters slots [c_begin, c_end) (one CTA's chunk).  tot_e / pre_e
// give expert e's total count and the count in earlier chunks (thread e < E
// calls them); CTA `writer` also writes counts and offsets.
template <typename Tot, typename Pre>
__device__ __forceinline__ void permute_rank_scatter(const int32_t *__restrict__ ids, int c_begin, int c_end, int E,
                                                     Tot tot_e, Pre pre_e, bool writer, int32_t *counts,
                                                     int32_t *offsets, int32_t *sorted_slot, int32_t *dest_pos,
                                                     int32_t *s_mem)
{
    int32_t *s_base = s_mem;                                  // [E] next position of each expert in this chunk
    int32_t *s_scan = s_mem + E;                              // [kPermThreads] scan scratch
    uint16_t *s_wcnt = (uint16_t *)(s_scan + kPermThreads);   // [32 warps][E]
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

    // expert totals, this chunk's prefix, and the exclusive scan over experts
    // (warp shuffles, then one warp over the 32 warp totals)
    int tot = 0, pre = 0;
    if (tid < E) {
        tot = tot_e(tid);
        pre = pre_e(tid);
    }
    int incl = tot;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off)
            incl += n;
    }
    if (lane == 31)
        s_scan[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int wsum = s_scan[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int n = __shfl_up_sync(0xFFFFFFFFu, wsum, off);
            if (lane >= off)
                wsum += n;
        }
        s_scan[32 + lane] = wsum;   // inclusive prefix of the warp totals
    }
    __syncthreads();
    incl += warp > 0 ? s_scan[32 + warp - 1] : 0;
    if (tid < E) {
        const int off_e = incl - tot;
        s_base[tid] = off_e + pre;
        if (writer) {
            counts[tid] = tot;
            offsets[tid] = off_e;
        }
    }
    if (writer && tid == 0)
        offsets[E] = s_scan[32 + 31];
    for (int i = tid; i < 32 * E; i += kPermThreads)
        s_wcnt[i] = 0;
    __syncthreads();

    for (int c0 = c_begin; c0 < c_end; c0 += kPermThreads) {
        const int s = c0 + tid;
        int e = -1;
        if (s < c_end) {
            e = ids[s];
            if (e < 0 || e >= E)
                e = -1;
        }
        const uint32_t peers = __match_any_sync(0xFFFFFFFFu, e);
        const int rank_w = __popc(peers & ((1u << lane) - 1u));
        if (e >= 0 && lane == __ffs(peers) - 1)
            s_wcnt[warp * E + e] = (uint16_t)__popc(peers);
        __syncthreads();
        if (e >= 0) {
            int rank = s_base[e] + rank_w;
            for (int w = 0; w < warp; ++w)
                rank += s_wcnt[w * E + e];
            sorted_slot[rank] = s;
            dest_pos[s] = rank;
        } else if (s < c_end) {
            dest_pos[s] = -1;
        }
        __syncthreads();
        // advance the per-expert positions past this sub-chunk, clear the counts
        for (int ee = tid; ee < E; ee += kPermThreads) {
            int add = 0;
            for (int w = 0; w < 32; ++w) {
                add += s_wcnt[w * E + ee];
                s_wcnt[w * E + ee] = 0;
            }
            s_base[ee] += add;
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kPermThreads) permute_scatter_kernel(const int32_t *__restrict__ ids, int S, int E,
                                                                       int chunk, const int32_t *__restrict__ hist,
                                                                       int32_t *counts, int32_t *offsets,
                                                                       int32_t *sorted_slot, int32_t *dest_pos)
{
    pdl_wait();
    pdl_allow_successor();
    extern __shared__ int32_t s_mem[];
    const int nblk = gridDim.x, b = blockIdx.x;
    auto tot_e = [&](int e) {
        int t = 0;
        for (int bb = 0; bb < nblk; ++bb)
            t += hist[(size_t)bb * E + e];
        return t;
    };
    auto pre_e = [&](int e) {
        int t = 0;
        for (int bb = 0; bb < b; ++bb)
            t += hist[(size_t)bb * E + e];
        return t;
    };
    permute_rank_scatter(ids, b * chunk, min(S, (b + 1) * chunk), E, tot_e, pre_e, b == 0, counts, offsets,
                         sorted_slot, dest_pos, s_mem);
}

// Small problems (up to two 1024-slot passes): histogram, scan and scatter in
// one CTA and one launch.  Larger ones spread the slots over several CTAs.
constexpr int kPermSingleMax = 2048;

__global__ void __launch_bounds__(kPermThreads) permute_single_kernel(const int32_t *__restrict__ ids, int S, int E,
                                                                      int32_t *counts, int32_t *offsets,
                                                                      int32_t *sorted_slot, int32_t *dest_pos,
                                                                      int *status)
{
    pdl_wait();
    pdl_allow_successor();
    extern __shared__ int32_t s_mem[];
    int32_t *s_hist = s_mem + E + kPermThreads + (32 * E + 1) / 2;   // [E], after the scatter's scratch
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        s_hist[e] = 0;
    __syncthreads();
    for (int s = threadIdx.x; s < S; s += blockDim.x) {
        const int e = ids[s];
        if (e >= 0 && e < E)
            atomicAdd(&s_hist[e], 1);
        else
            record_error(status, MOE_ERR_INVALID_ARG, s);
    }
    __syncthreads();
    permute_rank_scatter(ids, 0, S, E, [&](int e) { return s_hist[e]; }, [](int) { return 0; }, true, counts,
                         offsets, sorted_slot, dest_pos, s_mem);
}

int permute_launch_count(int T, int k) { return T * k == 0 ? 0 : (T * k <= kPermSingleMax ? 1 : 2); }

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
    if (S <= kPermSingleMax) {
        const size_t smem1 = (E + kPermThreads) * sizeof(int32_t) + ((32 * E + 1) / 2) * sizeof(int32_t) +
                             E * sizeof(int32_t);
        if (smem1 > 48 * 1024) {
            const cudaError_t e1 =
                cudaFuncSetAttribute(permute_single_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
            if (e1 != cudaSuccess)
                return e1;
        }
        return launch_pdl(permute_single_kernel, 1, kPermThreads, smem1, st, ids, S, E, counts, offsets, sorted_slot,
                          dest_pos, status);
    }
    const int chunk = perm_chunk(S);
    const int nblk = perm_blocks(S);
    int32_t *hist = (int32_t *)scratch;
    cudaError_t err =
        launch_pdl(permute_hist_kernel, nblk, kPermThreads, E * sizeof(int32_t), st, ids, S, E, chunk, hist, status);
    if (err != cudaSuccess)
        return err;
    const size_t smem = (E + kPermThreads) * sizeof(int32_t) + 32 * E * sizeof(uint16_t);
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(permute_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess)
            return err;
    }
    return launch_pdl(permute_scatter_kernel, nblk, kPermThreads, smem, st, ids, S, E, chunk, (const int32_t *)hist,
                      counts, offsets, sorted_slot, dest_pos);
}


// ------------------------------------------------------------------------
// Token rows in permuted order: out[p] = x[sorted_slot[p] / k] for the
// rows p < rows, then the shared expert's rows out[rows + t] = x[t] for
// t < shared_rows, so that the gate/up GEMM can read each expert's rows as
// one contiguous block with TMA tiles.  One warp copies one row with
// 16-byte vectors (H a multiple of 128).  In the fp16-operand mode each
// bf16 value is written as fp16 (exact for 2^-17 <= |x| <= 65504, rounded
// below); a value beyond fp16's range records MOE_ERR_UNSUPPORTED.
// ------------------------------------------------------------------------

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v, bool &bad)
{
    const float lo = __uint_as_float(v << 16), hi = __uint_as_float(v & 0xFFFF0000u);
    bad |= !(fabsf(lo) <= 65504.f) || !(fabsf(hi) <= 65504.f);
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t *__restrict__ x,
                                                          const int32_t *__restrict__ sorted_slot, int rows,
                                                          int shared_rows, int k, int H, int to_f16,
                                                          uint16_t *__restrict__ out, int *status)
{
    pdl_wait();
    pdl_allow_successor();
    const int lane = threadIdx.x & 31;
    const int n16 = H / 8;
    const int warps = gridDim.x * (blockDim.x / 32);
    bool bad = false;
    for (int p = (blockIdx.x * blockDim.x + threadIdx.x) / 32; p < rows + shared_rows; p += warps) {
        const int t = p < rows ? sorted_slot[p] / k : p - rows;
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * H);
        uint4 *dst = reinterpret_cast<uint4 *>(out + (size_t)p * H);
        // four 16-byte loads per lane in flight before their stores
        for (int i0 = lane; i0 < n16; i0 += 4 * 32) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (i0 + 32 * u < n16)
                    v[u] = src[i0 + 32 * u];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (i0 + 32 * u >= n16)
                    break;
                if (to_f16) {
                    v[u].x = bf16x2_to_f16x2(v[u].x, bad);
                    v[u].y = bf16x2_to_f16x2(v[u].y, bad);
                    v[u].z = bf16x2_to_f16x2(v[u].z, bad);
                    v[u].w = bf16x2_to_f16x2(v[u].w, bad);
                }
                dst[i0 + 32 * u] = v[u];
            }
        }
    }
    if (bad)
        record_error(status, MOE_ERR_UNSUPPORTED, 40);
}

cudaError_t launch_gather_rows(const uint16_t *x, const int32_t *sorted_slot, int rows, int k, int H, uint16_t *out,
                               int num_sms, cudaStream_t st, int shared_rows, bool to_f16, int *status)
{
    const int total = rows + shared_rows;
    if (total <= 0)
        return cudaSuccess;
    const int need = (total + 7) / 8;   // eight warps per block
    const int blocks = need < 4 * num_sms ? need : 4 * num_sms;
    return launch_pdl(gather_rows_kernel, blocks, 256, 0, st, x, sorted_slot, rows, shared_rows, k, H,
                      to_f16 ? 1 : 0, out, status);
}

// ------------------------------------------------------------------------
// Allocation-free variant of moe_permute.
//
// Some callers cannot allocate device memory at the point where they need a
// permutation: code running inside another allocator's critical section, a
// plugin host that forbids cudaMalloc after start-up, or a caller that has no
// workspace to hand over.  For them the chunk histograms live in one
// fixed-size array in device global memory that belongs to this library.
// Its size bounds the expert count (E <= kNoAllocMaxExperts); the token count
// is not bounded by it, because the slots are always cut into at most 32
// chunks.  Every GPU that loads the library keeps the array until the process
// exits.
//
// The array is shared by all calls on a device: two calls that overlap on the
// GPU (different streams without ordering between them) race on it.  Each
// call rewrites every histogram entry it later reads, so nothing has to be
// cleared between calls.
// ------------------------------------------------------------------------

constexpr int kNoAllocMaxExperts = 1024;
static __device__ __align__(256) int32_t g_noalloc_hist[kPermMaxChunks * kNoAllocMaxExperts];

// Device address of g_noalloc_hist, looked up once per device (the name
// alone is a host-side stand-in, not a device address).
static int32_t *noalloc_hist_ptr(cudaError_t *err)
{
    static std::mutex mu;
    static int32_t *ptrs[64] = {nullptr};
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess)
        return nullptr;
    if (dev < 0 || dev >= 64) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_noalloc_hist);
        if (*err != cudaSuccess)
            return nullptr;
        ptrs[dev] = (int32_t *)p;
    }
    return ptrs[dev];
}

int noalloc_max_experts() { return kNoAllocMaxExperts; }

cudaError_t launch_permute_noalloc(const int32_t *ids, int T, int E, int k, int32_t *counts, int32_t *offsets,
                                   int32_t *sorted_slot, int32_t *dest_pos, cudaStream_t st)
{
    const int S = T * k;
    if (S == 0) {
        cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, st);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st);
        return e;
    }
    cudaError_t err = cudaSuccess;
    int32_t *hist = noalloc_hist_ptr(&err);
    if (!hist)
        return err;
    const int chunk = perm_chunk(S);
    const int nblk = perm_blocks(S);
    // ids outside [0, E) are not reported through a status word here; their
    // dest_pos entries come back as -1
    err = launch_pdl(permute_hist_kernel, nblk, kPermThreads, E * sizeof(int32_t), st, ids, S, E, chunk, hist,
                     (int *)nullptr);
    if (err != cudaSuccess)
        return err;
    const size_t smem = (E + kPermThreads) * sizeof(int32_t) + 32 * E * sizeof(uint16_t);
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(permute_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess)
            return err;
    }
    return launch_pdl(permute_scatter_kernel, nblk, kPermThreads, smem, st, ids, S, E, chunk, (const int32_t *)hist,
                      counts, offsets, sorted_slot, dest_pos);
}

}  // namespace moeq4
