// Fused decode layer: the whole MoE layer for a handful of tokens in one
// cooperative kernel.
//
// With T <= 8 tokens the layer reads a few experts (k per token plus the
// shared one) and does little arithmetic, so a chain of separate kernels
// spends most of its time in launch gaps and pipeline fill.  Here one CTA
// per SM runs four phases separated by two grid barriers (bounded waits):
//
//   A  router: logits[t, e] = x[t] . Wr[e] (+ bias), gate[t] = x[t] . g;
//      one warp per router row, rows spread over the CTAs
//   B  every CTA routes all T tokens itself (top-k as in route.cu) and
//      groups the (token, expert) pairs by expert
//   C  gate/up + SwiGLU: a unit is (expert, 16 features), i.e. 16 rows of
//      Wg and the 16 matching rows of Wu, one row per lane; the 16 warps
//      split K = H, and the next unit's codes are loaded while the current
//      one is computed:  h[p, i] = silu(x[t] . Wg_e[i]) * (x[t] . Wu_e[i])
//   D  down and combine: a unit is 16 output columns of every chosen
//      expert; lanes split K = I, and the combine of those columns happens
//      in the same CTA:  y[t, c] = bf16( sum_j w[t,j] (h[p(t,j)] . Wd_e[c])
//                                         + sigmoid(gate[t]) (h[shared t] . Wd_s[c]) )
//
// The expert weights stay in the packed 4-bit layout of dequant.cuh.  Each
// 32-weight chunk is decoded to its integer codes (exact small integers in
// fp32) and the dot product is taken against the codes; the chunk's scale
// and offset are applied once per chunk:  sum_i (a u_i + b) x_i =
// a (sum_i u_i x_i) + b (sum_i x_i).  The weights so used are the exact
// dequantised values of the format (the GEMM path rounds them to bf16 for
// the tensor cores), and no intermediate is rounded to bf16 before y.
//
// Each phase runs its code a few times per launch at most, so instruction
// fetch is a large share of its time: loops over tokens, chunks and units
// stay rolled, and the kernel is instantiated per weight format.
//
// Work is split by output rows and columns with fixed K slices, and every
// sum runs in a fixed order, so the result does not depend on the number of
// CTAs.
#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "decode.h"
#include "dequant.cuh"
#include "kernels.h"
#include "ptx.cuh"

#ifdef MOEQ4_TRACE
// phase timestamps (%globaltimer) of the first four CTAs, thread 0
__device__ unsigned long long g_dec_trace[4][16];
#define DEC_MARK(i)                                                   \
    do {                                                              \
        if (blockIdx.x < 4 && threadIdx.x == 0)                       \
            g_dec_trace[blockIdx.x][(i)] = moeq4::globaltimer_ns();    \
    } while (0)
#else
#define DEC_MARK(i) \
    do {            \
    } while (0)
#endif

namespace moeq4 {

namespace {

constexpr int kThreads = kDecodeThreads;
constexpr int kWarps = kThreads / 32;
constexpr int kN = kDecodeMaxT;
constexpr int kPad = 36;    // floats per 32-element chunk row in shared memory (bank spread)
constexpr int kFeat = 16;   // features per gate/up unit: 16 gate rows + 16 up rows, one per lane
constexpr int kCols = 16;   // output columns per down unit
constexpr int kDnBatch = 8; // down: slot passes whose codes are in flight at once

__device__ __forceinline__ unsigned ld_acquire(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned ld_relaxed(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(unsigned *p, unsigned v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Grid barrier over all CTAs of a cooperative launch.  bar[0] counts
// arrivals (back to 0 after every barrier), bar[1] is the generation,
// bar[2] the abort flag.  Waits are bounded by the workspace's wait budget
// (status word 20, microseconds; 0 = 2 s): on timeout the CTA records
// MOE_ERR_TIMEOUT, raises the abort flag (so the others stop waiting) and
// the caller returns.  Returns false when the kernel must stop.
//
// Test knob (status word 21): when it holds c > 0, CTA c - 1 waits at the
// first barrier without arriving, so that every CTA's wait runs out of its
// budget (the way a lost arrival would); the kernel then returns with
// MOE_ERR_TIMEOUT and a usable context.
__device__ bool grid_sync(unsigned *bar, int *status, int where, int *s_flag)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 1;
        __threadfence();
        const unsigned gen = ld_acquire(bar + 1);   // read before arriving: it cannot move until we do
        const bool skip = where == 91 && test_knob_hits_this_cta(status);
        const unsigned prev = skip ? 0u : atomicAdd(bar, 1u);
        if (!skip && prev == gridDim.x - 1) {
            atomicExch(bar, 0u);
            __threadfence();
            st_release(bar + 1, gen + 1);
        } else {
            const uint64_t t0 = globaltimer_ns(), limit = wait_limit_ns(status);
            uint32_t spins = 0;
            while (ld_acquire(bar + 1) == gen) {
                if (ld_relaxed(bar + 2)) {
                    ok = 0;
                    break;
                }
                if ((++spins & 63u) == 0 && globaltimer_ns() - t0 > limit) {
                    atomicExch(bar + 2, 1u);
                    record_error(status, MOE_ERR_TIMEOUT, where);
                    ok = 0;
                    break;
                }
            }
        }
        __threadfence();
        *s_flag = ok;
    }
    __syncthreads();
    return *s_flag != 0;
}

__device__ __forceinline__ bool better(float v, int id, float bv, int bid)
{
    return v > bv || (v == bv && id < bid);
}

// (a, b) of one 32-weight chunk so that weight_i = a * c_i + b, where c_i
// is the decoded code: q = u - 8 for int4-sym (b = 0), u for the others.
// gshift: log2 of the int4 group size.
template <int WFMT>
__device__ __forceinline__ void chunk_coeffs(const uint8_t *mblock, int m, int ngroups, int r, int kpos, int gshift,
                                             float &a, float &b)
{
    if (WFMT == MOE_WFMT_Q4K) {
        const int sb = kpos >> 8;
        const uint4 hdr = __ldg((const uint4 *)(mblock + ((size_t)(m * ngroups + sb) * kTileRows + r) * 16));
        float dsc, dm;
        q4k_subblock_scale(hdr, (kpos & 255) >> 5, dsc, dm);
        a = dsc;
        b = -dm;
    } else if (WFMT == MOE_WFMT_INT4_ASYM) {
        const uint32_t sm =
            __ldg((const uint32_t *)(mblock + ((size_t)(m * ngroups + (kpos >> gshift)) * kTileRows + r) * 4));
        a = __uint_as_float(sm << 16);
        b = __uint_as_float(sm & 0xFFFF0000u);
    } else {
        const uint16_t s =
            __ldg((const uint16_t *)(mblock + ((size_t)(m * ngroups + (kpos >> gshift)) * kTileRows + r) * 2));
        a = __uint_as_float((uint32_t)s << 16);
        b = 0.f;
    }
}

// 32 codes of a chunk -> their integer values in fp32, element order.
// Element 8w + 2i sits in nibble i of word w, element 8w + 2i + 1 in
// nibble i + 4.  Two codes at a time become a bf16 pair 128 + u (exact),
// minus 136 (int4-sym: q = u - 8) or 128 (the others), both exact.
template <bool SYM>
__device__ __forceinline__ void decode_codes(const uint4 codes, float (&c)[32])
{
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
    const uint32_t off = SYM ? 0x43084308u : 0x43004300u;
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t t = bf16x2_sub(((w[wi] >> (4 * i)) & 0x000F000Fu) | 0x43004300u, off);
            c[8 * wi + 2 * i] = __uint_as_float(t << 16);
            c[8 * wi + 2 * i + 1] = __uint_as_float(t & 0xFFFF0000u);
        }
    }
}

// sum_i c_i v_i over one padded 32-float row in shared memory, four
// independent partial sums added in a fixed order
__device__ __forceinline__ float dot32(const float (&c)[32], const float *v)
{
    float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 x4 = *(const float4 *)(v + 4 * q);
        p0 = fmaf(c[4 * q], x4.x, p0);
        p1 = fmaf(c[4 * q + 1], x4.y, p1);
        p2 = fmaf(c[4 * q + 2], x4.z, p2);
        p3 = fmaf(c[4 * q + 3], x4.w, p3);
    }
    return (p0 + p1) + (p2 + p3);
}

// sum of the 32 floats of a padded chunk row, in order
__device__ __forceinline__ float chunk_sum(const float *p)
{
    float s = 0.f;
    for (int q = 0; q < 32; ++q)
        s += p[q];
    return s;
}

// Top-k of one token by one warp (lane l holds logits l, l + 32, ...):
// ties to the lower id, weights softmax over the kept k (renorm) or over
// all E.  Lane j < k returns the j-th id and weight; a position left
// unfilled (NaN logits) returns id -1.
template <int NPL>
__device__ __forceinline__ void topk_warp(const float *Lrow, int E, int k, int renorm, int lane, int &my_id,
                                          float &my_w)
{
    float v[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = i * 32 + lane;
        v[i] = e < E ? __ldcg(Lrow + e) : -CUDART_INF_F;
    }
    uint32_t taken = 0;
    float top = 0.f, my_val = 0.f;
    my_id = -1;
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
        if (bid != 0x7FFFFFFF && (bid & 31) == lane)
            taken |= 1u << (bid >> 5);
        if (j == 0)
            top = bv;
        if (lane == j) {
            my_val = bv;
            my_id = bid == 0x7FFFFFFF ? -1 : bid;
        }
    }
    const float ex = lane < k ? expf(my_val - top) : 0.f;
    float z;
    if (renorm) {
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
    my_w = ex / z;
}

// Codes and chunk coefficients of one gate/up unit, this thread's share:
// lane = row (gate rows 0-15, up rows 16-31 of the unit's 16 features),
// chunks j = warp + 16 n of K = H (n < 4; H <= 2048 per pass of j0).
struct GuLoad {
    uint4 cd[4];
    float ca[4], cb[4];
};

template <int WFMT>
__device__ __forceinline__ void gu_load(const DecodeArgs &A, int e, int f0, int j0, int nchH, int ngroups, int gshift,
                                        int warp, int lane, GuLoad &g)
{
    const int F = A.I / kTileRows, KS = A.H / kKStep;
    const int m = lane >> 4, R = f0 + (lane & 15);
    const size_t tile = (size_t)e * F + R / kTileRows;
    const int r = R % kTileRows;
    const uint8_t *qb = A.gu_q + tile * KS * code_block_bytes(2) + ((size_t)m * 2 * kTileRows + r) * kChunkBytes;
    const uint8_t *mb = A.gu_meta + tile * A.gu_meta_bytes;
#pragma unroll
    for (int n = 0; n < 4; ++n) {
        const int j = j0 + warp + n * kWarps;
        if (j < nchH) {
            g.cd[n] = __ldg((const uint4 *)(qb + (size_t)(j >> 1) * code_block_bytes(2) +
                                            (size_t)(j & 1) * kTileRows * kChunkBytes));
            chunk_coeffs<WFMT>(mb, m, ngroups, r, j * 32, gshift, g.ca[n], g.cb[n]);
        } else {
            g.cd[n] = make_uint4(0, 0, 0, 0);
            g.ca[n] = g.cb[n] = 0.f;
        }
    }
}

}  // namespace

DecodeSmem decode_smem_layout(int T, int k, int H, int I, int has_shared)
{
    DecodeSmem s{};
    const int tk = T * k;
    const int np = tk + (has_shared ? T : 0);
    const int nd = tk + (has_shared ? 1 : 0);
    const size_t xrows = (size_t)T * (H / 32), hrows = (size_t)np * (I / 32);
    const size_t rows = xrows > hrows ? xrows : hrows;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += (bytes + 15) & ~(size_t)15;
        return (int)o;
    };
    s.big = take(sizeof(float) * kPad * rows);
    s.sums = take(sizeof(float) * rows);
    // gate/up partials [warp][token][lane]; reused for the down outputs [pair][column]
    const size_t red = (size_t)kWarps * kN * 32 > (size_t)np * kCols ? (size_t)kWarps * kN * 32 : (size_t)np * kCols;
    s.red = take(sizeof(float) * red);
    s.ids = take(sizeof(int) * (tk > 0 ? tk : 1));
    s.w = take(sizeof(float) * np);
    s.pidx = take(sizeof(int) * (tk > 0 ? tk : 1));
    s.pair_tok = take(sizeof(int) * np);
    s.pair_w = take(sizeof(float) * np);
    s.slot_e = take(sizeof(int) * nd);
    s.slot_base = take(sizeof(int) * nd);
    s.slot_cnt = take(sizeof(int) * nd);
    s.bitmap = take(sizeof(uint32_t) * 32);
    s.wprefix = take(sizeof(int) * 33);
    s.flag = take(sizeof(int) * 4);
    s.bytes = off;
    return s;
}

namespace {

template <int WFMT>
__global__ void __launch_bounds__(kThreads, 1) decode_layer_kernel(const DecodeArgs A, const DecodeSmem L)
{
    extern __shared__ __align__(16) uint8_t smem[];
    float *big = (float *)(smem + L.big);
    float *sums = (float *)(smem + L.sums);
    float *red = (float *)(smem + L.red);
    int *ids_s = (int *)(smem + L.ids);
    float *w_s = (float *)(smem + L.w);
    int *pidx = (int *)(smem + L.pidx);
    int *pair_tok = (int *)(smem + L.pair_tok);
    float *pair_w = (float *)(smem + L.pair_w);
    int *slot_e = (int *)(smem + L.slot_e);
    int *slot_base = (int *)(smem + L.slot_base);
    int *slot_cnt = (int *)(smem + L.slot_cnt);
    uint32_t *bitmap = (uint32_t *)(smem + L.bitmap);
    int *wprefix = (int *)(smem + L.wprefix);
    int *flag = (int *)(smem + L.flag);

    constexpr bool kSym = WFMT == MOE_WFMT_INT4_SYM;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = A.T, H = A.H, I = A.I, E = A.E, k = A.k;
    const int tk = T * k;
    const int nchH = H / 32, nchI = I / 32;
    const int gshift = __ffs(A.G > 0 ? A.G : 1) - 1;

    // a previous launch on this workspace gave up in a barrier: stop before touching it
    if (ld_relaxed(A.bar + 2)) {
        if (blockIdx.x == 0 && tid == 0)
            record_error(A.status, MOE_ERR_TIMEOUT, 90);
        return;
    }
    DEC_MARK(0);
    if (tid < 32)
        bitmap[tid] = 0;

    // ------------------------------------------------ A: x -> smem, router
    {
        for (int i = tid; i < T * (H / 8); i += kThreads) {
            const int t = i / (H / 8), kk = (i % (H / 8)) * 8;
            const uint4 v = *(const uint4 *)(A.x + (size_t)t * H + kk);
            float *dst = big + ((size_t)t * nchH + kk / 32) * kPad + kk % 32;
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
            *(float4 *)dst = make_float4(__uint_as_float(u[0] << 16), __uint_as_float(u[0] & 0xFFFF0000u),
                                         __uint_as_float(u[1] << 16), __uint_as_float(u[1] & 0xFFFF0000u));
            *(float4 *)(dst + 4) = make_float4(__uint_as_float(u[2] << 16), __uint_as_float(u[2] & 0xFFFF0000u),
                                               __uint_as_float(u[3] << 16), __uint_as_float(u[3] & 0xFFFF0000u));
        }
        __syncthreads();
        for (int i = tid; i < T * nchH; i += kThreads)
            sums[i] = chunk_sum(big + (size_t)i * kPad);
        // one warp per router row (and the shared gate vector); a lane holds
        // 16 float4 of a 2048-wide slice of the row, loaded before any use
        float *racc = red + warp * kN;
        const int rows = E + (A.has_shared ? 1 : 0);
        for (int e = blockIdx.x + gridDim.x * warp; e < rows; e += gridDim.x * kWarps) {
            const float *wrow = e < E ? A.router_w + (size_t)e * H : A.shared_gate;
            for (int seg = 0; seg < H; seg += 2048) {
                float4 wv[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int kk = seg + (q * 32 + lane) * 4;
                    wv[q] = kk < H ? __ldg((const float4 *)(wrow + kk)) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
                for (int t = 0; t < T; ++t) {
                    const float *xt = big + (size_t)t * nchH * kPad;
                    float a0 = 0.f, a1 = 0.f;
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const int kk = seg + (q * 32 + lane) * 4;
                        if (kk < H) {
                            const float4 xv = *(const float4 *)(xt + (kk / 32) * kPad + kk % 32);
                            a0 = fmaf(wv[q].x, xv.x, a0);
                            a1 = fmaf(wv[q].y, xv.y, a1);
                            a0 = fmaf(wv[q].z, xv.z, a0);
                            a1 = fmaf(wv[q].w, xv.w, a1);
                        }
                    }
                    float v = a0 + a1;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)
                        v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
                    if (lane == 0)
                        racc[t] = seg == 0 ? v : racc[t] + v;
                }
            }
            __syncwarp();
            if (lane < T) {
                const float s = racc[lane];
                if (e < E)
                    A.logits[(size_t)lane * E + e] = A.router_bias ? s + A.router_bias[e] : s;
                else
                    A.gate_logit[lane] = s;
            }
            __syncwarp();
        }
    }
    DEC_MARK(1);
    if (!grid_sync(A.bar, A.status, 91, flag))
        return;
    DEC_MARK(2);

    // ------------------------------------------------ B: routing, pair lists
    if (warp < T) {
        const int t = warp;
        int my_id = 0;
        float my_w = 0.f;
        if (A.override_ids) {
            if (lane < k) {
                my_id = A.override_ids[(size_t)t * k + lane];
                my_w = A.override_w[(size_t)t * k + lane];
            }
        } else if (E <= 256) {
            topk_warp<8>(A.logits + (size_t)t * E, E, k, A.renorm, lane, my_id, my_w);
        } else {
            topk_warp<32>(A.logits + (size_t)t * E, E, k, A.renorm, lane, my_id, my_w);
        }
        if (lane < k) {
            // an id outside [0, E) (given, or none found among NaN logits) is
            // reported and its slot carries expert 0 with weight 0
            if (my_id < 0 || my_id >= E) {
                if (blockIdx.x == 0)
                    record_error(A.status, MOE_ERR_INVALID_ARG, t * k + lane);
                my_id = 0;
                my_w = 0.f;
            }
            ids_s[t * k + lane] = my_id;
            w_s[t * k + lane] = my_w;
        }
        if (lane == 0 && A.has_shared)
            w_s[tk + t] = 1.0f / (1.0f + expf(-__ldcg(A.gate_logit + t)));
    }
    __syncthreads();
    if (blockIdx.x == 0) {
        for (int i = tid; i < tk; i += kThreads) {
            A.topk_ids[i] = ids_s[i];
            A.topk_w[i] = w_s[i];
        }
    }
    for (int i = tid; i < tk; i += kThreads)
        atomicOr(&bitmap[ids_s[i] >> 5], 1u << (ids_s[i] & 31));
    __syncthreads();
    if (warp == 0) {
        const int c = __popc(bitmap[lane]);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o)
                incl += n;
        }
        wprefix[lane] = incl - c;
        if (lane == 31)
            wprefix[32] = incl;
    }
    __syncthreads();
    // pair p of (t, j): pairs ordered by expert, then by t k + j
    for (int i = tid; i < tk; i += kThreads) {
        const int e = ids_s[i];
        int below = 0, before = 0, same = 0;
        for (int i2 = 0; i2 < tk; ++i2) {
            const int e2 = ids_s[i2];
            below += e2 < e;
            same += e2 == e;
            before += (e2 == e) & (i2 < i);
        }
        const int p = below + before;
        const int d = wprefix[e >> 5] + __popc(bitmap[e >> 5] & ((1u << (e & 31)) - 1u));
        pair_tok[p] = i / k;
        pair_w[p] = w_s[i];
        pidx[i] = p;
        if (before == 0) {
            slot_e[d] = e;
            slot_base[d] = below;
            slot_cnt[d] = same;
        }
    }
    const int nd_routed = wprefix[32];
    if (A.has_shared) {
        for (int t = tid; t < T; t += kThreads) {
            pair_tok[tk + t] = t;
            pair_w[tk + t] = w_s[tk + t];
        }
        if (tid == 0) {
            slot_e[nd_routed] = E;
            slot_base[nd_routed] = tk;
            slot_cnt[nd_routed] = T;
        }
    }
    __syncthreads();
    const int Nd = nd_routed + (A.has_shared ? 1 : 0);
    const int NP = tk + (A.has_shared ? T : 0);
    DEC_MARK(3);

    // ------------------------------------------------ C: gate/up + SwiGLU
    {
        const int ngroups = WFMT == MOE_WFMT_Q4K ? H / 256 : H >> gshift;
        const int per_slot = I / kFeat;
        const int U = Nd * per_slot;
        float *part = red;   // [warp][token][lane]
        GuLoad cur, nxt;
        int u = blockIdx.x;
        if (u < U)
            gu_load<WFMT>(A, slot_e[u / per_slot], (u % per_slot) * kFeat, 0, nchH, ngroups, gshift, warp, lane, cur);
        for (; u < U; u += gridDim.x) {
            const int d = u / per_slot, f0 = (u % per_slot) * kFeat;
            const int base = slot_base[d], cnt = slot_cnt[d];
            for (int i = 0; i < cnt; ++i)
                part[(warp * kN + i) * 32 + lane] = 0.f;
            for (int j0 = 0; j0 < nchH; j0 += 4 * kWarps) {
                // the next chunk group of this unit, or the first of the next unit
                const int jn = j0 + 4 * kWarps;
                const int un = u + gridDim.x;
                if (jn < nchH)
                    gu_load<WFMT>(A, slot_e[d], f0, jn, nchH, ngroups, gshift, warp, lane, nxt);
                else if (un < U)
                    gu_load<WFMT>(A, slot_e[un / per_slot], (un % per_slot) * kFeat, 0, nchH, ngroups, gshift, warp,
                                  lane, nxt);
                for (int i = 0; i < cnt; ++i) {
                    const int t = pair_tok[base + i];
                    float acc = 0.f;
#pragma unroll
                    for (int n = 0; n < 4; ++n) {
                        const int j = j0 + warp + n * kWarps;
                        if (j < nchH) {
                            float c[32];
                            decode_codes<kSym>(cur.cd[n], c);
                            const float dot = dot32(c, big + ((size_t)t * nchH + j) * kPad);
                            acc = fmaf(cur.ca[n], dot, fmaf(cur.cb[n], sums[t * nchH + j], acc));
                        }
                    }
                    part[(warp * kN + i) * 32 + lane] += acc;
                }
                cur = nxt;
            }
            __syncthreads();
            // feature f of the unit for its token i: gate and up sums over the warps, in order
            if (tid < kFeat * cnt) {
                const int i = tid / kFeat, f = tid % kFeat;
                float g = 0.f, v = 0.f;
                for (int w = 0; w < kWarps; ++w) {
                    g += part[(w * kN + i) * 32 + f];
                    v += part[(w * kN + i) * 32 + kFeat + f];
                }
                A.h[(size_t)(base + i) * I + f0 + f] = g / (1.0f + expf(-g)) * v;
            }
            __syncthreads();
        }
    }
    DEC_MARK(4);
    if (!grid_sync(A.bar, A.status, 92, flag))
        return;
    DEC_MARK(5);

    // ------------------------------------------------ D: down + combine
    {
        float *hs = big;
        for (int i = tid; i < NP * (I / 4); i += kThreads) {
            const int p = i / (I / 4), kk = (i % (I / 4)) * 4;
            const float4 v = __ldcg((const float4 *)(A.h + (size_t)p * I + kk));
            *(float4 *)(hs + ((size_t)p * nchI + kk / 32) * kPad + kk % 32) = v;
        }
        __syncthreads();
        for (int i = tid; i < NP * nchI; i += kThreads)
            sums[i] = chunk_sum(hs + (size_t)i * kPad);
        __syncthreads();
        const int F = H / kTileRows, KS = I / kKStep, ngroups = WFMT == MOE_WFMT_Q4K ? I / 256 : I >> gshift;
        // lanes per row: the power of two >= I / 32 chunks (at most 32);
        // a slot pass covers kCols rows of one expert, SP passes side by side
        int LJ = 1;
        while (LJ < nchI)
            LJ <<= 1;
        const int per_pass = kCols * LJ;                // threads of one slot pass (>= 32: warp-uniform)
        const int SP = kThreads / per_pass;
        const int sub = tid / per_pass, cc = (tid / LJ) % kCols, j = tid % LJ;
        float *o_s = red;   // [pair][column]
        for (int u = blockIdx.x; u < H / kCols; u += gridDim.x) {
            const int C = u * kCols + cc;
            const int r = C % kTileRows;
            for (int d0 = 0; d0 < Nd; d0 += SP * kDnBatch) {
                uint4 cd[kDnBatch];
                float ca[kDnBatch], cb[kDnBatch];
#pragma unroll
                for (int b = 0; b < kDnBatch; ++b) {
                    const int d = d0 + b * SP + sub;
                    cd[b] = make_uint4(0, 0, 0, 0);
                    ca[b] = cb[b] = 0.f;
                    if (d < Nd && j < nchI) {
                        const size_t tile = (size_t)slot_e[d] * F + C / kTileRows;
                        cd[b] = __ldg((const uint4 *)(A.dn_q + (tile * KS + (j >> 1)) * code_block_bytes(1) +
                                                      ((size_t)(j & 1) * kTileRows + r) * kChunkBytes));
                        chunk_coeffs<WFMT>(A.dn_meta + tile * A.dn_meta_bytes, 0, ngroups, r, j * 32, gshift, ca[b],
                                           cb[b]);
                    }
                }
#pragma unroll
                for (int b = 0; b < kDnBatch; ++b) {
                    const int d = d0 + b * SP + sub;
                    if (d >= Nd)
                        continue;   // uniform over the pass's threads, which span whole warps
                    const int base = slot_base[d], cnt = slot_cnt[d];
                    float c[32];
                    decode_codes<kSym>(cd[b], c);
                    for (int i = 0; i < cnt; ++i) {
                        const int p = base + i;
                        float v = 0.f;
                        if (j < nchI)
                            v = fmaf(ca[b], dot32(c, hs + ((size_t)p * nchI + j) * kPad), cb[b] * sums[p * nchI + j]);
                        for (int o = LJ >> 1; o > 0; o >>= 1)
                            v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
                        if (j == 0)
                            o_s[p * kCols + cc] = v;
                    }
                }
            }
            __syncthreads();
            // the combine of these columns: routed experts in j order, then the shared expert
            if (tid < T * kCols) {
                const int t = tid / kCols, c2 = tid % kCols;
                float acc = 0.f;
                for (int jj = 0; jj < k; ++jj)
                    acc = fmaf(w_s[t * k + jj], o_s[pidx[t * k + jj] * kCols + c2], acc);
                if (A.has_shared)
                    acc = fmaf(w_s[tk + t], o_s[(tk + t) * kCols + c2], acc);
                A.y[(size_t)t * H + u * kCols + c2] = (uint16_t)(pack_bf16x2(acc, 0.f) & 0xFFFFu);
            }
            __syncthreads();
        }
    }
    DEC_MARK(6);
}

}  // namespace

cudaError_t launch_decode_layer(const DecodeArgs &a, int grid, cudaStream_t st)
{
    const DecodeSmem L = decode_smem_layout(a.T, a.k, a.H, a.I, a.has_shared);
    void (*kern)(const DecodeArgs, const DecodeSmem) =
        a.wfmt == MOE_WFMT_Q4K         ? decode_layer_kernel<MOE_WFMT_Q4K>
        : a.wfmt == MOE_WFMT_INT4_ASYM ? decode_layer_kernel<MOE_WFMT_INT4_ASYM>
                                       : decode_layer_kernel<MOE_WFMT_INT4_SYM>;
    // the opt-in limit once per device and format (callers never ask for
    // more: see the admission check)
    static std::atomic<bool> configured[64][3];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    const int f = a.wfmt == MOE_WFMT_Q4K ? 1 : a.wfmt == MOE_WFMT_INT4_ASYM ? 2 : 0;
    if (dev < 0 || dev >= 64 || !configured[dev][f].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess)
            return e;
        if (dev >= 0 && dev < 64)
            configured[dev][f].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = L.bytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;   // all CTAs resident at once, or the launch fails
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a, L);
}

}  // namespace moeq4

#ifdef MOEQ4_TRACE
extern "C" int moe_decode_trace_fetch(unsigned long long *host)
{
    return (int)cudaMemcpyFromSymbol(host, g_dec_trace, sizeof(g_dec_trace));
}
#endif
