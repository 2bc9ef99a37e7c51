// Fused decode layer: the whole MoE layer for a handful of tokens in one
// cooperative kernel.
//
// With T <= 8 tokens the layer reads a few experts (k per token plus the
// shared one) and does little arithmetic, so a chain of separate kernels
// spends most of its time in launch gaps and pipeline fill.  Here one CTA
// per SM runs five phases separated by grid barriers (bounded waits):
//
//   A  router: logits[t, e] = x[t] . Wr[e] (+ bias), gate[t] = x[t] . g
//      (fp32 FMAs on CUDA cores; rows of Wr spread over the CTAs)
//   B  every CTA routes all T tokens itself (top-k as in route.cu), groups
//      the (token, expert) pairs by expert and starts L2 prefetches of the
//      chosen experts' weights
//   C  gate/up + SwiGLU: one warp per (expert, 4 rows of I), full K = H:
//      h[p, i] = silu(x[t] . Wg_e[i]) * (x[t] . Wu_e[i])   (fp32)
//   D  down: one warp per (expert, 4 rows of H), full K = I:
//      o[p, j] = h[p] . Wd_e[j]                              (fp32)
//   E  combine: y[t] = bf16( sum_j w[t,j] o[p(t,j)] + sigmoid(gate[t]) o[shared t] )
//
// The expert weights stay in the packed 4-bit layout of dequant.cuh.  Each
// 32-weight chunk is decoded to its integer codes (exact small integers in
// fp32) and the dot product is taken against the codes; the chunk's scale
// and offset are applied once per chunk:  sum_i (a u_i + b) x_i =
// a (sum_i u_i x_i) + b (sum_i x_i).  The weights so used are the exact
// dequantised values of the format (the GEMM path rounds them to bf16 for
// the tensor cores), and no intermediate is rounded to bf16 before y.
//
// Work is split by output rows, never by K, and every sum runs in a fixed
// order, so the result does not depend on the number of CTAs.
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
__device__ unsigned long long g_dec_trace[4][10];
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
constexpr int kPad = 36;           // floats per 32-element chunk row in shared memory (bank spread)
constexpr int kPrefetchBytes = 32768;

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

__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Grid barrier over all CTAs of a cooperative launch.  bar[0] counts
// arrivals (back to 0 after every barrier), bar[1] is the generation,
// bar[2] the abort flag.  Waits are bounded by the workspace's wait budget
// (status word 20, microseconds; 0 = 2 s): on timeout the CTA records
// MOE_ERR_TIMEOUT, raises the abort flag (so the others stop waiting) and
// the caller returns.  Returns false when the kernel must stop.
//
// Test knob, status word 21: when it holds c > 0, CTA c - 1 waits at the
// first barrier without arriving, so that every CTA's wait runs out of its
// budget (the way a lost arrival would); the kernel then returns with
// MOE_ERR_TIMEOUT and a usable context.
constexpr int kStatusSkipArrivalWord = 21;

__device__ bool grid_sync(unsigned *bar, int *status, int where, int *s_flag)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 1;
        __threadfence();
        const unsigned gen = ld_acquire(bar + 1);   // read before arriving: it cannot move until we do
        const bool skip = where == 91 && status &&
                          *(const volatile int *)(status + kStatusSkipArrivalWord) == (int)blockIdx.x + 1;
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
__device__ __forceinline__ void chunk_coeffs(const DecodeArgs &A, const uint8_t *mblock, int m, int ngroups, int r,
                                             int kpos, float &a, float &b)
{
    if (A.wfmt == MOE_WFMT_Q4K) {
        const int sb = kpos / 256;
        const uint4 hdr = *(const uint4 *)(mblock + ((size_t)(m * ngroups + sb) * kTileRows + r) * 16);
        float dsc, dm;
        q4k_subblock_scale(hdr, (kpos % 256) / 32, dsc, dm);
        a = dsc;
        b = -dm;
    } else if (A.wfmt == MOE_WFMT_INT4_ASYM) {
        const uint32_t sm = *(const uint32_t *)(mblock + ((size_t)(m * ngroups + kpos / A.G) * kTileRows + r) * 4);
        a = __uint_as_float(sm << 16);
        b = __uint_as_float(sm & 0xFFFF0000u);
    } else {
        const uint16_t s = *(const uint16_t *)(mblock + ((size_t)(m * ngroups + kpos / A.G) * kTileRows + r) * 2);
        a = __uint_as_float((uint32_t)s << 16);
        b = 0.f;
    }
}

// 32 codes of a chunk -> their integer values in fp32, element order.
// Element 8w + 2i sits in nibble i of word w, element 8w + 2i + 1 in
// nibble i + 4.  Two codes at a time become a bf16 pair 128 + u (exact),
// minus 136 (int4-sym: q = u - 8) or 128 (the others), both exact.
__device__ __forceinline__ void decode_codes(const uint4 codes, bool sym, float (&c)[32])
{
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
    const uint32_t off = sym ? 0x43084308u : 0x43004300u;
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

// sum_i c_i v_i over one padded 32-float row in shared memory
__device__ __forceinline__ float dot32(const float (&c)[32], const float *v)
{
    float acc = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 x4 = *(const float4 *)(v + 4 * q);
        acc = fmaf(c[4 * q], x4.x, acc);
        acc = fmaf(c[4 * q + 1], x4.y, acc);
        acc = fmaf(c[4 * q + 2], x4.z, acc);
        acc = fmaf(c[4 * q + 3], x4.w, acc);
    }
    return acc;
}

// L2 prefetch of the weights of `nslots` experts, piece q of all pieces
// handled by thread (q mod grid threads); slot_e(d) gives the expert.
template <typename SlotE>
__device__ void prefetch_experts(const DecodeArgs &A, int nslots, SlotE slot_e)
{
    const size_t gu_codes = (size_t)(A.I / kTileRows) * (A.H / kKStep) * code_block_bytes(2);
    const size_t gu_meta = (size_t)(A.I / kTileRows) * A.gu_meta_bytes;
    const size_t dn_codes = (size_t)(A.H / kTileRows) * (A.I / kKStep) * code_block_bytes(1);
    const size_t dn_meta = (size_t)(A.H / kTileRows) * A.dn_meta_bytes;
    auto pieces = [](size_t b) { return (int)((b + kPrefetchBytes - 1) / kPrefetchBytes); };
    const int n0 = pieces(gu_codes), n1 = pieces(gu_meta), n2 = pieces(dn_codes), n3 = pieces(dn_meta);
    const int pps = n0 + n1 + n2 + n3;
    const int total = nslots * pps;
    for (int q = blockIdx.x + gridDim.x * threadIdx.x; q < total; q += gridDim.x * blockDim.x) {
        const size_t e = (size_t)slot_e(q / pps);
        int w = q % pps;
        const uint8_t *base;
        size_t size;
        if (w < n0) {
            base = A.gu_q + e * gu_codes;
            size = gu_codes;
        } else if ((w -= n0) < n1) {
            base = A.gu_meta + e * gu_meta;
            size = gu_meta;
        } else if ((w -= n1) < n2) {
            base = A.dn_q + e * dn_codes;
            size = dn_codes;
        } else {
            w -= n2;
            base = A.dn_meta + e * dn_meta;
            size = dn_meta;
        }
        const size_t off = (size_t)w * kPrefetchBytes;
        const size_t left = size - off;
        prefetch_l2(base + off, (uint32_t)(left < (size_t)kPrefetchBytes ? left : (size_t)kPrefetchBytes));
    }
}

}  // namespace

DecodeSmem decode_smem_layout(int T, int k, int H, int I, int has_shared)
{
    DecodeSmem s{};
    const int tk = T * k;
    const int np = tk + (has_shared ? T : 0);
    const int nd = tk + (has_shared ? 1 : 0);
    const size_t big = (size_t)kPad * ((size_t)T * (H / 32) > (size_t)np * (I / 32) ? (size_t)T * (H / 32)
                                                                                        : (size_t)np * (I / 32));
    const size_t sums = (size_t)T * (H / 32) > (size_t)np * (I / 32) ? (size_t)T * (H / 32) : (size_t)np * (I / 32);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += (bytes + 15) & ~(size_t)15;
        return (int)o;
    };
    s.big = take(sizeof(float) * big);
    s.sums = take(sizeof(float) * sums);
    s.red = take(sizeof(float) * kWarps * kDecodeMaxT);
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

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = A.T, H = A.H, I = A.I, E = A.E, k = A.k;
    const int tk = T * k;
    const int nchH = H / 32, nchI = I / 32;
    const bool sym = A.wfmt == MOE_WFMT_INT4_SYM;

    // a previous launch on this workspace gave up in a barrier: stop before touching it
    if (ld_relaxed(A.bar + 2)) {
        if (blockIdx.x == 0 && tid == 0)
            record_error(A.status, MOE_ERR_TIMEOUT, 90);
        return;
    }
    DEC_MARK(0);
    if (tid < 32)
        bitmap[tid] = 0;

    // the shared expert is known in advance: start its prefetch now
    if (A.has_shared)
        prefetch_experts(A, 1, [&](int) { return E; });

    // ------------------------------------------------ A: x -> smem, router
    {
        float *xs = big;
        for (int i = tid; i < T * H / 8; i += kThreads) {
            const int t = i / (H / 8), kk = (i % (H / 8)) * 8;
            const uint4 v = *(const uint4 *)(A.x + (size_t)t * H + kk);
            float *dst = xs + (size_t)t * nchH * kPad + (kk / 32) * kPad + kk % 32;
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
            *(float4 *)dst = make_float4(__uint_as_float(u[0] << 16), __uint_as_float(u[0] & 0xFFFF0000u),
                                         __uint_as_float(u[1] << 16), __uint_as_float(u[1] & 0xFFFF0000u));
            *(float4 *)(dst + 4) = make_float4(__uint_as_float(u[2] << 16), __uint_as_float(u[2] & 0xFFFF0000u),
                                               __uint_as_float(u[3] << 16), __uint_as_float(u[3] & 0xFFFF0000u));
        }
        __syncthreads();
        // chunk sums of x (the offset term of asymmetric formats)
        for (int i = tid; i < T * nchH; i += kThreads) {
            const float *src = xs + (size_t)i * kPad;
            float s = 0.f;
            for (int q = 0; q < 32; ++q)
                s += src[q];
            sums[i] = s;
        }
        const int rows = E + (A.has_shared ? 1 : 0);
        for (int e = blockIdx.x; e < rows; e += gridDim.x) {
            const float *wrow = e < E ? A.router_w + (size_t)e * H : A.shared_gate;
            float part[kDecodeMaxT];
#pragma unroll
            for (int t = 0; t < kDecodeMaxT; ++t)
                part[t] = 0.f;
            for (int q = tid; q < H / 4; q += kThreads) {
                const float4 wv = __ldg((const float4 *)wrow + q);
                const int kk = 4 * q;
                const float *xp = xs + (kk / 32) * kPad + kk % 32;
#pragma unroll
                for (int t = 0; t < kDecodeMaxT; ++t) {
                    if (t < T) {
                        const float4 xv = *(const float4 *)(xp + (size_t)t * nchH * kPad);
                        float a = part[t];
                        a = fmaf(wv.x, xv.x, a);
                        a = fmaf(wv.y, xv.y, a);
                        a = fmaf(wv.z, xv.z, a);
                        a = fmaf(wv.w, xv.w, a);
                        part[t] = a;
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < kDecodeMaxT; ++t) {
                float v = part[t];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
                if (lane == 0 && t < T)
                    red[warp * kDecodeMaxT + t] = v;
            }
            __syncthreads();
            if (tid < T) {
                float s = 0.f;
                for (int w = 0; w < kWarps; ++w)
                    s += red[w * kDecodeMaxT + tid];
                if (e < E)
                    A.logits[(size_t)tid * E + e] = A.router_bias ? s + A.router_bias[e] : s;
                else
                    A.gate_logit[tid] = s;
            }
            __syncthreads();
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
        } else {
            constexpr int NPL = 32;   // E <= 1024
            const int npl = (E + 31) / 32;
            float v[NPL];
            const float *Lrow = A.logits + (size_t)t * E;
#pragma unroll
            for (int i = 0; i < NPL; ++i) {
                const int e = i * 32 + lane;
                v[i] = (i < npl && e < E) ? __ldcg(Lrow + e) : -CUDART_INF_F;
            }
            uint32_t taken = 0;
            float top = 0.f, my_val = 0.f;
            for (int j = 0; j < k; ++j) {
                float bv = -CUDART_INF_F;
                int bid = 0x7FFFFFFF;
#pragma unroll
                for (int i = 0; i < NPL; ++i) {
                    const int e = i * 32 + lane;
                    if (i < npl && e < E && !((taken >> i) & 1u) && better(v[i], e, bv, bid)) {
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
                if (bid < E && (bid & 31) == lane)
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
            if (A.renorm) {
                z = 0.f;
                for (int j = 0; j < k; ++j)
                    z += __shfl_sync(0xFFFFFFFFu, ex, j);
            } else {
                float part = 0.f;
#pragma unroll
                for (int i = 0; i < NPL; ++i)
                    if (i < npl && i * 32 + lane < E)
                        part += expf(v[i] - top);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
                    part += __shfl_xor_sync(0xFFFFFFFFu, part, off);
                z = part;
            }
            my_w = ex / z;
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
    prefetch_experts(A, nd_routed, [&](int d) { return slot_e[d]; });

    // ------------------------------------------------ C: gate/up + SwiGLU
    {
        const float *xs = big;
        const int F = I / kTileRows, KS = H / kKStep, ngroups = A.wfmt == MOE_WFMT_Q4K ? H / 256 : H / A.G;
        const int r4 = lane & 3, jp = lane >> 2;
        const int units = Nd * (I / 4);
        for (int u = blockIdx.x + gridDim.x * warp; u < units; u += gridDim.x * kWarps) {
            const int d = u / (I / 4), row0 = (u % (I / 4)) * 4;
            const int e = slot_e[d], base = slot_base[d], cnt = slot_cnt[d];
            const size_t tile = (size_t)e * F + row0 / kTileRows;
            const int r = row0 % kTileRows + r4;
            const uint8_t *qb = A.gu_q + tile * KS * code_block_bytes(2) + (size_t)r * kChunkBytes;
            const uint8_t *mb = A.gu_meta + tile * A.gu_meta_bytes;
            for (int i0 = 0; i0 < cnt; i0 += kDecodeMaxT) {
                float acc[2][kDecodeMaxT];
#pragma unroll
                for (int m = 0; m < 2; ++m)
#pragma unroll
                    for (int i = 0; i < kDecodeMaxT; ++i)
                        acc[m][i] = 0.f;
                for (int j0 = 0; j0 < nchH; j0 += 32) {
                    // up to four chunks of this lane, both matrices: loads first
                    uint4 cd[4][2];
                    float ca[4][2], cb[4][2];
#pragma unroll
                    for (int n = 0; n < 4; ++n) {
                        const int j = j0 + jp + 8 * n;
#pragma unroll
                        for (int m = 0; m < 2; ++m) {
                            if (j < nchH) {
                                cd[n][m] = __ldg((const uint4 *)(qb + ((size_t)((j >> 1) * 2 + m) * 2 + (j & 1)) *
                                                                          kTileRows * kChunkBytes));
                                chunk_coeffs(A, mb, m, ngroups, r, j * 32, ca[n][m], cb[n][m]);
                            } else {
                                cd[n][m] = make_uint4(0, 0, 0, 0);
                                ca[n][m] = cb[n][m] = 0.f;
                            }
                        }
                    }
#pragma unroll
                    for (int n = 0; n < 4; ++n) {
                        const int j = j0 + jp + 8 * n;
                        if (j >= nchH)
                            continue;
#pragma unroll
                        for (int m = 0; m < 2; ++m) {
                            float c[32];
                            decode_codes(cd[n][m], sym, c);
#pragma unroll
                            for (int i = 0; i < kDecodeMaxT; ++i) {
                                if (i0 + i < cnt) {
                                    const int t = pair_tok[base + i0 + i];
                                    const float dot = dot32(c, xs + ((size_t)t * nchH + j) * kPad);
                                    acc[m][i] = fmaf(ca[n][m], dot, fmaf(cb[n][m], sums[t * nchH + j], acc[m][i]));
                                }
                            }
                        }
                    }
                }
#pragma unroll
                for (int m = 0; m < 2; ++m)
#pragma unroll
                    for (int i = 0; i < kDecodeMaxT; ++i)
#pragma unroll
                        for (int o = 4; o < 32; o <<= 1)
                            acc[m][i] += __shfl_xor_sync(0xFFFFFFFFu, acc[m][i], o);
                if (jp == 0) {
#pragma unroll
                    for (int i = 0; i < kDecodeMaxT; ++i) {
                        if (i0 + i < cnt) {
                            const float g = acc[0][i];
                            A.h[(size_t)(base + i0 + i) * I + row0 + r4] = g / (1.0f + expf(-g)) * acc[1][i];
                        }
                    }
                }
            }
        }
    }
    DEC_MARK(4);
    if (!grid_sync(A.bar, A.status, 92, flag))
        return;
    DEC_MARK(5);

    // ------------------------------------------------ D: down
    {
        float *hs = big;
        for (int i = tid; i < NP * I / 4; i += kThreads) {
            const int p = i / (I / 4), kk = (i % (I / 4)) * 4;
            const float4 v = __ldcg((const float4 *)(A.h + (size_t)p * I + kk));
            *(float4 *)(hs + ((size_t)p * nchI + kk / 32) * kPad + kk % 32) = v;
        }
        __syncthreads();
        for (int i = tid; i < NP * nchI; i += kThreads) {
            const float *src = hs + (size_t)i * kPad;
            float s = 0.f;
            for (int q = 0; q < 32; ++q)
                s += src[q];
            sums[i] = s;
        }
        __syncthreads();
        const int F = H / kTileRows, KS = I / kKStep, ngroups = A.wfmt == MOE_WFMT_Q4K ? I / 256 : I / A.G;
        const int r4 = lane & 3, jp = lane >> 2;
        const int units = Nd * (H / 4);
        for (int u = blockIdx.x + gridDim.x * warp; u < units; u += gridDim.x * kWarps) {
            const int d = u / (H / 4), row0 = (u % (H / 4)) * 4;
            const int e = slot_e[d], base = slot_base[d], cnt = slot_cnt[d];
            const size_t tile = (size_t)e * F + row0 / kTileRows;
            const int r = row0 % kTileRows + r4;
            const uint8_t *qb = A.dn_q + tile * KS * code_block_bytes(1) + (size_t)r * kChunkBytes;
            const uint8_t *mb = A.dn_meta + tile * A.dn_meta_bytes;
            for (int i0 = 0; i0 < cnt; i0 += kDecodeMaxT) {
                float acc[kDecodeMaxT];
#pragma unroll
                for (int i = 0; i < kDecodeMaxT; ++i)
                    acc[i] = 0.f;
                for (int j0 = 0; j0 < nchI; j0 += 32) {
                    uint4 cd[4];
                    float ca[4], cb[4];
#pragma unroll
                    for (int n = 0; n < 4; ++n) {
                        const int j = j0 + jp + 8 * n;
                        if (j < nchI) {
                            cd[n] = __ldg((const uint4 *)(qb + ((size_t)(j >> 1) * 2 + (j & 1)) * kTileRows *
                                                                   kChunkBytes));
                            chunk_coeffs(A, mb, 0, ngroups, r, j * 32, ca[n], cb[n]);
                        } else {
                            cd[n] = make_uint4(0, 0, 0, 0);
                            ca[n] = cb[n] = 0.f;
                        }
                    }
#pragma unroll
                    for (int n = 0; n < 4; ++n) {
                        const int j = j0 + jp + 8 * n;
                        if (j >= nchI)
                            continue;
                        float c[32];
                        decode_codes(cd[n], sym, c);
#pragma unroll
                        for (int i = 0; i < kDecodeMaxT; ++i) {
                            if (i0 + i < cnt) {
                                const int p = base + i0 + i;
                                const float dot = dot32(c, hs + ((size_t)p * nchI + j) * kPad);
                                acc[i] = fmaf(ca[n], dot, fmaf(cb[n], sums[p * nchI + j], acc[i]));
                            }
                        }
                    }
                }
#pragma unroll
                for (int i = 0; i < kDecodeMaxT; ++i)
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1)
                        acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], o);
                if (jp == 0) {
#pragma unroll
                    for (int i = 0; i < kDecodeMaxT; ++i)
                        if (i0 + i < cnt)
                            A.o[(size_t)(base + i0 + i) * H + row0 + r4] = acc[i];
                }
            }
        }
    }
    DEC_MARK(6);
    if (!grid_sync(A.bar, A.status, 93, flag))
        return;
    DEC_MARK(7);

    // ------------------------------------------------ E: combine
    for (int i = blockIdx.x * kThreads + tid; i < T * H; i += gridDim.x * kThreads) {
        const int t = i / H, col = i % H;
        float acc = 0.f;
        for (int j = 0; j < k; ++j)
            acc = fmaf(w_s[t * k + j], __ldcg(A.o + (size_t)pidx[t * k + j] * H + col), acc);
        if (A.has_shared)
            acc = fmaf(w_s[tk + t], __ldcg(A.o + (size_t)(tk + t) * H + col), acc);
        A.y[i] = (uint16_t)(pack_bf16x2(acc, 0.f) & 0xFFFFu);
    }
    DEC_MARK(8);
}

cudaError_t launch_decode_layer(const DecodeArgs &a, int grid, cudaStream_t st)
{
    const DecodeSmem L = decode_smem_layout(a.T, a.k, a.H, a.I, a.has_shared);
    // the opt-in limit once per device (callers never ask for more: see the admission check)
    static std::atomic<bool> configured[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64 || !configured[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(decode_layer_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess)
            return e;
        if (dev >= 0 && dev < 64)
            configured[dev].store(true, std::memory_order_release);
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
    return cudaLaunchKernelEx(&cfg, decode_layer_kernel, a, L);
}

}  // namespace moeq4

#ifdef MOEQ4_TRACE
extern "C" int moe_decode_trace_fetch(unsigned long long *host)
{
    return (int)cudaMemcpyFromSymbol(host, g_dec_trace, sizeof(g_dec_trace));
}
#endif
