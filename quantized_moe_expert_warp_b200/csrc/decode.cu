// Fused decode layer: the whole MoE layer for a handful of tokens in one
// cooperative kernel.
//
// With T <= 8 tokens the layer reads a few experts (k per token plus the
// shared one) and does little arithmetic, so a chain of separate kernels
// spends most of its time in launch gaps and pipeline fill.  Here one CTA
// per SM runs four phases separated by two grid barriers (bounded waits):
//
//   A  router: logits[t, e] = x[t] . Wr[e] (+ bias), gate[t] = x[t] . g;
//      one warp per router row (fp32 FMAs), rows spread over the CTAs
//   B  every CTA routes all T tokens itself (top-k as in route.cu) and
//      groups the (token, expert) pairs by expert, in slots of at most 8
//      pairs (the columns of one MMA)
//   C  gate/up + SwiGLU: a unit is (slot, 16 features), i.e. a 16-row tile
//      of Wg and the matching tile of Wu; the 16 warps split K = H, each
//      runs warp-level m16n8k16 tensor-core MMAs against the slot's tokens
//      (up to 8 columns), and the warps' sums are added in a fixed order:
//          h[p, i] = bf16( silu(x[t] . Wg_e[i]) * (x[t] . Wu_e[i]) )
//   D  down and combine: a unit is 16 output columns (a 16-row tile of Wd)
//      of every slot, one warp per slot, MMAs against the slot's h rows;
//      the combine of those columns happens in the CTA:
//          y[t, c] = bf16( sum_j w[t,j] (h[p(t,j)] . Wd_e[c])
//                          + sigmoid(gate[t]) (h[shared t] . Wd_s[c]) )
//
// The expert weights stay in the packed 4-bit layout of dequant.cuh and are
// staged per warp in shared memory with cp.async (a ring of 2 to 4 items,
// so that later items' codes are in flight during the current one).  An MMA's A operand is
// built straight from the codes: one shift and one logical op give the bf16
// pair (128 + u, 128 + u') of two codes, exact.  Each 32-weight chunk's scale
// and offset are applied to the fp32 MMA result once per chunk,
//     sum_i (a c_i + b) v_i = a (sum_i (128 + u_i) v_i - o sum_i v_i) + b sum_i v_i,
// with c_i = u_i - 8, o = 136 (int4-sym) or c_i = u_i, o = 128 (the others),
// so the weights enter at their exact dequantised values; x is bf16 (exact)
// and h is rounded to bf16 once, as on the prefill path.
//
// The chunks of one staged item are unrolled so that their MMA chains
// overlap; loops over tokens, items and units stay rolled, which keeps the
// code that runs once per launch small, and the kernel is instantiated per
// weight format.
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
#include "topk.cuh"

#ifdef MOEQ4_TRACE
// phase timestamps (%globaltimer) of the first four CTAs, thread 0
__device__ unsigned long long g_dec_trace[4][24];
#define DEC_MARK(i)                                                   \
    do {                                                              \
        if (blockIdx.x < 4 && threadIdx.x == 0)                       \
            g_dec_trace[blockIdx.x][(i)] = moeq4::globaltimer_ns();    \
    } while (0)
// entries 7 .. 10: steps inside the routing phase; 11 .. 14: warp 0's
// cycles in the gate/up phase issuing copies, waiting for them, in the MMA
// loop and in the hand-off; 15: warp 0's cycles waiting for its staged down
// items; 16, 17: clock64 at the start and the end of the gate/up phase
#define DEC_CLK(v) const long long v = clock64()
#define DEC_ACC(a, since) (a) += clock64() - (since)
#define DEC_DECL(a) long long a = 0
#else
#define DEC_MARK(i) \
    do {            \
    } while (0)
#define DEC_CLK(v)
#define DEC_ACC(a, since)
#define DEC_DECL(a)
#endif

namespace moeq4 {

namespace {

constexpr int kThreads = kDecodeThreads;
constexpr int kWarps = kThreads / 32;
constexpr int kN = kDecodeMaxT;
constexpr int kFeat = 16;   // features per gate/up unit: 16 gate rows + 16 up rows, one per lane
constexpr int kCols = 16;   // output columns per down unit
constexpr int kCodeBuf = 2048; // staged codes of one warp item
// row stride (floats) of the 16-wide rows of the gate/up partials and the
// down outputs in shared memory: 20 puts the 4 column pairs a warp's MMA
// fragment writes on distinct banks
constexpr int kRedLd = 20;
// bytes of one row's scale entry: bf16 scale (int4-sym), bf16 scale and
// minimum (int4-asym), 16-byte super-block header (Q4K)
__host__ __device__ constexpr int meta_row_bytes(int wfmt)
{
    return wfmt == MOE_WFMT_Q4K ? 16 : wfmt == MOE_WFMT_INT4_ASYM ? 4 : 2;
}
// one warp item: its codes, then the scale entries of its 16 rows for each
// of its 8 (chunk, matrix) pairs
__host__ __device__ constexpr int item_buf_bytes(int wfmt) { return kCodeBuf + 8 * 16 * meta_row_bytes(wfmt); }

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

// Grid barrier over all CTAs of a cooperative launch.  bar[0] is the
// arrival word: CTA 0 adds 2^31 - (n - 1) and every other CTA adds 1, so
// its top bit flips exactly when the last of the n CTAs arrives and its low
// bits come back to where they were (no reset step, and one atomic on the
// critical path); a CTA waits for the flip relative to the word it saw when
// it arrived.  bar[2] is the abort flag.  Waits are bounded by wait_ns (the
// workspace's wait budget, status word 20, microseconds; 0 = 2 s): on
// timeout the CTA records MOE_ERR_TIMEOUT, raises the abort flag (so the
// others stop waiting) and the caller returns.  Returns false when the
// kernel must stop.  Only thread 0's skip and wait_ns are read.
//
// Test knob (status word 21): when it holds c > 0, CTA c - 1 waits at the
// first barrier without arriving (skip), so that every CTA's wait runs out
// of its budget (the way a lost arrival would); the kernel then returns
// with MOE_ERR_TIMEOUT and a usable context.
__device__ bool grid_sync(unsigned *bar, int *status, int where, int *s_flag, bool skip, uint64_t wait_ns)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 1;
        __threadfence();   // this CTA's global writes before its arrival
        const unsigned add = blockIdx.x == 0 ? 0x80000000u - (gridDim.x - 1) : 1u;
        const unsigned seen = skip ? ld_acquire(bar) : atomicAdd(bar, add);
        if (skip || (((seen + add) ^ seen) & 0x80000000u) == 0) {   // not the last arrival
            const uint64_t t0 = globaltimer_ns();
            uint32_t spins = 0;
            while (((ld_acquire(bar) ^ seen) & 0x80000000u) == 0) {
                if (ld_relaxed(bar + 2)) {
                    ok = 0;
                    break;
                }
                if ((++spins & 63u) == 0 && globaltimer_ns() - t0 > wait_ns) {
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


// (a, b) of one 32-weight chunk so that weight_i = a * c_i + b, where c_i
// is the decoded code (q = u - 8 for int4-sym with b = 0, u for the
// others), from the row's staged scale entry; kpos is the chunk's first
// position along K.
template <int WFMT>
__device__ __forceinline__ void staged_coeffs(const uint8_t *mrow, int kpos, float &a, float &b)
{
    if (WFMT == MOE_WFMT_Q4K) {
        float dsc, dm;
        q4k_subblock_scale(*(const uint4 *)mrow, (kpos & 255) >> 5, dsc, dm);
        a = dsc;
        b = -dm;
    } else if (WFMT == MOE_WFMT_INT4_ASYM) {
        const uint32_t sm = *(const uint32_t *)mrow;
        a = __uint_as_float(sm << 16);
        b = __uint_as_float(sm & 0xFFFF0000u);
    } else if (WFMT == MOE_WFMT_INT4_SYM_F16) {
        a = __half2float(__ushort_as_half(*(const uint16_t *)mrow));
        b = 0.f;
    } else {
        a = __uint_as_float((uint32_t) * (const uint16_t *)mrow << 16);
        b = 0.f;
    }
}

// 32-weight chunks that share one scale entry, capped at 4 (the chunks one
// warp takes together): G / 32 for the int4 formats, 1 for Q4K (its
// sub-block scales change every 32 weights).
template <int WFMT>
__device__ __forceinline__ int chunks_per_group(int G)
{
    if (WFMT == MOE_WFMT_Q4K)
        return 1;
    return G >= 128 ? 4 : G >= 64 ? 2 : 1;
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
    float top, my_val;
    warp_topk<NPL>(v, E, k, lane, my_val, my_id, top);
    if (my_id == 0x7FFFFFFF)
        my_id = -1;
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

// Warp-level bf16 MMA, m16n8k16, fp32 accumulate: d += A B.  A: 16 x 16
// (row), B: 16 x 8 (col); lane = 4 gid + tid4 holds A rows gid and gid + 8,
// B column gid, D rows gid, gid + 8 and columns 2 tid4, 2 tid4 + 1.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The bf16 pair (128 + u_{2i}, 128 + u_{2i+1}) of nibbles i and i + 4 of a
// code word (exact values): the A-fragment register for columns 2i, 2i + 1.
__device__ __forceinline__ uint32_t code_pair(uint32_t w, int i)
{
    return ((w >> (4 * i)) & 0x000F000Fu) | 0x43004300u;
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// cp.async.wait_group with a run-time count (0 .. 3)
__device__ __forceinline__ void cp_async_wait_upto(int n)
{
    if (n >= 3)
        cp_async_wait_group<3>();
    else if (n == 2)
        cp_async_wait_group<2>();
    else if (n == 1)
        cp_async_wait_group<1>();
    else
        cp_async_wait_group<0>();
}

// Rows 0 .. n - 1 of a row-major bf16 matrix (row length len, a multiple
// of 32) into shared rows of stride ld elements, then a zero row at shared
// row zrow: 16-byte cp.async (L2 only: the rows may have been written by
// other CTAs of this launch), all issued at once, as one commit group.
__device__ __forceinline__ void issue_rows(const uint16_t *src, int len, int n, int zrow, uint32_t dst, int ld,
                                           int tid)
{
    const int per_row = len / 8;
    for (int i = tid; i < (n + 1) * per_row; i += kThreads) {
        const int r = i / per_row, kk = (i % per_row) * 8;
        const bool real = r < n;
        cp_async_16(dst + 2u * (uint32_t)((real ? r : zrow) * ld + kk), real ? src + (size_t)r * len + kk : src,
                    real ? 16u : 0u);
    }
    cp_async_commit();
}

// The fp32 sum of every 32-element chunk of shared rows 0 .. n - 1 (stride
// ld) into sums[row][chunk].  Thread i reads 16 bytes (8 elements, summed
// in order; a warp reads consecutive bytes); the 4 threads of a chunk are
// consecutive lanes and add their parts with two shuffles.  The loop runs
// in whole warps so every shuffle is complete.
__device__ __forceinline__ void row_sums(const uint16_t *rows, int len, int n, int ld, float *sums, int tid)
{
    const int per_row = len / 8, nch = len / 32;
    const int rounded = (n * per_row + 31) & ~31;
    for (int i = tid; i < rounded; i += kThreads) {
        const int r = i / per_row, kk = (i % per_row) * 8;
        const uint4 v = r < n ? *(const uint4 *)(rows + (size_t)r * ld + kk) : make_uint4(0, 0, 0, 0);
        float s = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t w = word_of(v, q);
            s += __uint_as_float(w << 16);
            s += __uint_as_float(w & 0xFFFF0000u);
        }
        s += __shfl_xor_sync(0xFFFFFFFFu, s, 1);
        s += __shfl_xor_sync(0xFFFFFFFFu, s, 2);
        if (r < n && (i & 3) == 0)
            sums[(size_t)r * nch + kk / 32] = s;
    }
}

// One 32-element chunk of a 16-row tile against an 8-column B operand: the
// two k16 slices of the chunk.  lo / hi: this lane's codes of rows gid and
// gid + 8; brow: this lane's B column (a row of 16-bit values in shared
// memory) at the chunk's first element.
__device__ __forceinline__ void chunk_mma(float (&d)[4], const uint4 &lo, const uint4 &hi, const uint16_t *brow,
                                          int tid4)
{
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        const uint32_t a0 = code_pair(word_of(lo, 2 * s), tid4), a1 = code_pair(word_of(hi, 2 * s), tid4);
        const uint32_t a2 = code_pair(word_of(lo, 2 * s + 1), tid4), a3 = code_pair(word_of(hi, 2 * s + 1), tid4);
        const uint32_t b0 = *(const uint32_t *)(brow + 16 * s + 2 * tid4);
        const uint32_t b1 = *(const uint32_t *)(brow + 16 * s + 8 + 2 * tid4);
        mma_16816(d, a0, a1, a2, a3, b0, b1);
    }
}

}  // namespace

DecodeSmem decode_smem_layout(int T, int k, int H, int I, int has_shared, int wfmt)
{
    const int tk = T * k;
    const int np = tk + (has_shared ? T : 0);
    const int nd = tk + (has_shared ? 1 : 0);   // slots of at most 8 pairs: at most one per pair
    const int ntok = tk < kN ? (tk > 0 ? tk : 1) : kN;   // pairs (MMA columns) of one slot
    auto up16 = [](size_t b) { return (b + 15) & ~(size_t)15; };
    const size_t ring = (size_t)kWarps * item_buf_bytes(wfmt);
    auto build = [&](int nred) {
        DecodeSmem s{};
        size_t off = 0;
        auto take = [&](size_t bytes) {
            const size_t o = off;
            off += up16(bytes);
            return (int)o;
        };
        // phases A-C: x as bf16 rows (kN + 1, the last one zero) and its
        // chunk sums, then nred buffers of gate/up partials
        // [warp][matrix][pair < ntok][row] (the router's per-warp sums in
        // phase A use the first); phase D reuses the space for h (np + 1
        // rows), its chunk sums and the down outputs [pair][column]
        const size_t xbytes = up16(sizeof(uint16_t) * (size_t)(kN + 1) * (H + 8) + sizeof(float) * (size_t)kN * (H / 32));
        const size_t hbytes = up16(sizeof(uint16_t) * (size_t)(np + 1) * (I + 8) + sizeof(float) * (size_t)np * (I / 32));
        size_t redc = sizeof(float) * (size_t)kWarps * 2 * ntok * kRedLd;
        if ((size_t)nred * redc < sizeof(float) * kWarps * kN)
            redc = sizeof(float) * kWarps * kN;
        const size_t outd = up16(sizeof(float) * (size_t)np * kRedLd);
        s.big = take(xbytes + nred * redc > hbytes + outd ? xbytes + nred * redc : hbytes + outd);
        s.red = s.big + (int)xbytes;
        s.nred = nred;
        s.ntok = ntok;
        s.ored = s.big + (int)hbytes;
        s.ids = take(sizeof(int) * (tk > 0 ? tk : 1));
        s.w = take(sizeof(float) * np);
        s.pidx = take(sizeof(int) * (tk > 0 ? tk : 1));
        s.pair_tok = take(sizeof(int) * np);
        s.pair_w = take(sizeof(float) * np);
        s.slot_e = take(sizeof(int) * nd);
        s.slot_base = take(sizeof(int) * nd);
        s.slot_cnt = take(sizeof(int) * nd);
        // per chosen expert (rank d): its pairs per token (one byte per
        // token, 4 tokens a word), its expert id and its first pair
        s.tcount = take(sizeof(uint32_t) * 2 * (tk > 0 ? tk : 1));
        s.dexp = take(sizeof(int) * (tk > 0 ? tk : 1));
        s.dbase = take(sizeof(int) * (tk > 0 ? tk : 1));
        s.bitmap = take(sizeof(uint32_t) * 32);
        s.wprefix = take(sizeof(int) * 33);
        s.flag = take(sizeof(int) * 4);
        // the warps' staging rings take what is left, 2 to 4 items deep (a
        // shape whose 2-deep rings do not fit is refused by the caller)
        const size_t left = off < kDecodeSmemLimit ? kDecodeSmemLimit - off : 0;
        s.nstage = left / ring >= 4 ? 4 : left / ring >= 3 ? 3 : 2;
        s.cbuf = take(ring * s.nstage);
        s.bytes = off;
        return s;
    };
    // two partials buffers (one block barrier per gate/up unit) where they
    // fit beside 2-deep rings, else one (two barriers per unit)
    const DecodeSmem two = build(2);
    return two.bytes <= kDecodeSmemLimit ? two : build(1);
}

namespace {

// Gate/up staging of one unit pass for this warp, with 16-byte cp.async:
// chunks j = j0 + 4 warp + n (n < 4) of the 16 gate and 16 up rows of the
// unit, as codes [n][matrix][row][16 bytes] (2 KB), then the rows' scale
// entries of each (n, matrix) [n][matrix][row][entry].  gsh: log2 of the
// positions along K that share one entry.
template <int WFMT>
__device__ __forceinline__ void gu_stage(const DecodeArgs &A, int e, int f0, int j0, int nchH, int gsh, int warp,
                                         int lane, uint32_t dst)
{
    constexpr int MB = meta_row_bytes(WFMT);
    const int F = A.I / kTileRows, KS = A.H / kKStep;
    const int ngroups = A.H >> gsh;
    const size_t tile = (size_t)e * F + f0 / kTileRows;
    const int r0 = f0 % kTileRows;
    const uint8_t *mb = A.gu_meta + tile * A.gu_meta_bytes;
#pragma unroll
    for (int q = 0; q < (8 * MB + 31) / 32; ++q) {
        const int idx = lane + 32 * q;   // 8 MB pieces of 16 bytes
        if (idx < 8 * MB) {
            const int nm = idx / MB, pi = idx % MB, n = nm >> 1, m = nm & 1;
            const int j = j0 + 4 * warp + n;
            if (j < nchH) {
                const uint8_t *src = mb + ((size_t)(m * ngroups + ((j * 32) >> gsh)) * kTileRows + r0) * MB + 16 * pi;
                cp_async_16(dst + kCodeBuf + idx * 16, src, 16);
            }
        }
    }
    const uint8_t *base = A.gu_q + tile * KS * code_block_bytes(2);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int idx = lane + 32 * q;    // 128 pieces of 16 bytes
        const int n = idx >> 5, m = (idx >> 4) & 1, row = idx & 15;
        const int j = j0 + 4 * warp + n;
        if (j < nchH) {
            const uint8_t *src = base + (size_t)(j >> 1) * code_block_bytes(2) +
                                 ((size_t)(m * 2 + (j & 1)) * kTileRows + r0 + row) * kChunkBytes;
            cp_async_16(dst + idx * 16, src, 16);
        }
    }
}

// Down staging of one item for this warp: chunks j = 8 q + n (n < 8) of
// the 16 rows c0 .. c0 + 15 of expert e's down matrix, as codes
// [n][row][16 bytes] (2 KB), then the rows' scale entries [n][row][entry].
template <int WFMT>
__device__ __forceinline__ void dn_stage(const DecodeArgs &A, int e, int c0, int q, int nchI, int gsh, int lane,
                                         uint32_t dst)
{
    constexpr int MB = meta_row_bytes(WFMT);
    const int F = A.H / kTileRows, KS = A.I / kKStep;
    const size_t tile = (size_t)e * F + c0 / kTileRows;
    const int r0 = c0 % kTileRows;
    const uint8_t *mb = A.dn_meta + tile * A.dn_meta_bytes;
#pragma unroll
    for (int qq = 0; qq < (8 * MB + 31) / 32; ++qq) {
        const int idx = lane + 32 * qq;
        if (idx < 8 * MB) {
            const int n = idx / MB, pi = idx % MB;
            const int j = 8 * q + n;
            if (j < nchI) {
                const uint8_t *src = mb + ((size_t)((j * 32) >> gsh) * kTileRows + r0) * MB + 16 * pi;
                cp_async_16(dst + kCodeBuf + idx * 16, src, 16);
            }
        }
    }
    const uint8_t *base = A.dn_q + tile * KS * code_block_bytes(1);
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) {
        const int idx = lane + 32 * qq;
        const int n = idx >> 4, row = idx & 15;
        const int j = 8 * q + n;
        if (j < nchI) {
            const uint8_t *src = base + (size_t)(j >> 1) * code_block_bytes(1) +
                                 ((size_t)(j & 1) * kTileRows + r0 + row) * kChunkBytes;
            cp_async_16(dst + idx * 16, src, 16);
        }
    }
}

template <int WFMT>
__global__ void __launch_bounds__(kThreads, 1) decode_layer_kernel(const DecodeArgs A, const DecodeSmem L)
{
    extern __shared__ __align__(16) uint8_t smem[];
    float *red = (float *)(smem + L.red);
    uint8_t *cbuf = smem + L.cbuf;
    int *ids_s = (int *)(smem + L.ids);
    float *w_s = (float *)(smem + L.w);
    int *pidx = (int *)(smem + L.pidx);
    int *pair_tok = (int *)(smem + L.pair_tok);
    float *pair_w = (float *)(smem + L.pair_w);
    int *slot_e = (int *)(smem + L.slot_e);
    int *slot_base = (int *)(smem + L.slot_base);
    int *slot_cnt = (int *)(smem + L.slot_cnt);
    uint32_t *tcount = (uint32_t *)(smem + L.tcount);
    int *dexp = (int *)(smem + L.dexp);
    int *dbase = (int *)(smem + L.dbase);
    uint32_t *bitmap = (uint32_t *)(smem + L.bitmap);
    int *wprefix = (int *)(smem + L.wprefix);
    int *flag = (int *)(smem + L.flag);

    // code pair value minus the code
    constexpr float kOff = WFMT == MOE_WFMT_INT4_SYM || WFMT == MOE_WFMT_INT4_SYM_F16 ? 136.f : 128.f;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tid4 = lane & 3;
    const int T = A.T, H = A.H, I = A.I, E = A.E, k = A.k;
    const int tk = T * k;
    const int nchH = H / 32, nchI = I / 32;
    const int gshift = __ffs(A.G > 0 ? A.G : 1) - 1;
    // x as bf16 rows of H + 8 elements (row kN is zeros) and fp32 chunk sums
    const int XS = H + 8;
    uint16_t *xb = (uint16_t *)(smem + L.big);
    float *xsum = (float *)(xb + (size_t)(kN + 1) * XS);
    constexpr int kMB = meta_row_bytes(WFMT), kIB = item_buf_bytes(WFMT);
    const int NS = L.nstage;   // staging ring depth (items in flight per warp)
    uint8_t *mybuf = cbuf + (size_t)warp * NS * kIB;
    const uint32_t mybuf_s = smem_u32(mybuf);

    // the abort flag of a previous launch, and this warp's first router row,
    // are requested before anything else so that their latencies overlap
    const unsigned aborted = ld_relaxed(A.bar + 2);
    // rows t < T of x, then the zero row kN (rows T .. kN - 1 are never read)
    issue_rows(A.x, H, T, kN, smem_u32(xb), XS, tid);
    bool knob_skip = false;   // thread 0's barrier inputs, read early for the same reason
    uint64_t wait_ns = 0;
    if (tid == 0) {
        knob_skip = test_knob_hits_this_cta(A.status);
        wait_ns = wait_limit_ns(A.status);
    }
    const int rows = E + (A.has_shared ? 1 : 0);
    const int e_first = blockIdx.x + gridDim.x * warp;
    float4 wv[16];
    if (e_first < rows) {
        const float *wrow = e_first < E ? A.router_w + (size_t)e_first * H : A.shared_gate;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const int kk = (q * 32 + lane) * 4;
            wv[q] = kk < H ? __ldg((const float4 *)(wrow + kk)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    // a previous launch on this workspace gave up in a barrier: stop before touching it
    if (aborted) {
        cp_async_wait_group<0>();
        if (blockIdx.x == 0 && tid == 0)
            record_error(A.status, MOE_ERR_TIMEOUT, 90);
        return;
    }
    DEC_MARK(0);
    if (tid < 32)
        bitmap[tid] = 0;
    for (int i = tid; i < 2 * A.T * A.k; i += kThreads)
        tcount[i] = 0;

    // ------------------------------------------------ A: x -> smem, router
    {
        cp_async_wait_group<0>();
        __syncthreads();
        row_sums(xb, H, T, XS, xsum, tid);   // read in phase C, after two more block barriers
        // one warp per router row (and the shared gate vector); a lane holds
        // 16 float4 of a 2048-wide slice of the row, loaded before any use
        float *racc = red + warp * kN;
        for (int e = e_first; e < rows; e += gridDim.x * kWarps) {
            const float *wrow = e < E ? A.router_w + (size_t)e * H : A.shared_gate;
            for (int seg = 0; seg < H; seg += 2048) {
                if (e != e_first || seg != 0) {   // the first slice is already in registers
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const int kk = seg + (q * 32 + lane) * 4;
                        wv[q] = kk < H ? __ldg((const float4 *)(wrow + kk)) : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                }
                // two tokens against the slice at a time: 4 independent
                // chains, each summed in the same order as for one token
                for (int t0 = 0; t0 < T; t0 += 2) {
                    float a0[2] = {0.f, 0.f}, a1[2] = {0.f, 0.f};
                    const bool two = t0 + 1 < T;
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const int kk = seg + (q * 32 + lane) * 4;
                        if (kk < H) {
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                if (u == 0 || two) {
                                    const uint2 xv = *(const uint2 *)(xb + (size_t)(t0 + u) * XS + kk);
                                    a0[u] = fmaf(wv[q].x, __uint_as_float(xv.x << 16), a0[u]);
                                    a1[u] = fmaf(wv[q].y, __uint_as_float(xv.x & 0xFFFF0000u), a1[u]);
                                    a0[u] = fmaf(wv[q].z, __uint_as_float(xv.y << 16), a0[u]);
                                    a1[u] = fmaf(wv[q].w, __uint_as_float(xv.y & 0xFFFF0000u), a1[u]);
                                }
                            }
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        float v = a0[u] + a1[u];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1)
                            v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
                        if (lane == 0 && (u == 0 || two))
                            racc[t0 + u] = seg == 0 ? v : racc[t0 + u] + v;
                    }
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
    if (!grid_sync(A.bar, A.status, 91, flag, knob_skip, wait_ns))
        return;
    DEC_MARK(2);

    // ------------------------------------------------ B: routing, pair lists
    if (warp < T) {
        const int t = warp;
        // the shared expert's gate logit is requested with the logits
        const float glog = lane == 0 && A.has_shared ? __ldcg(A.gate_logit + t) : 0.f;
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
            w_s[tk + t] = 1.0f / (1.0f + expf(-glog));
    }
    DEC_MARK(7);
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
    DEC_MARK(8);
    // pair p of (t, j): pairs ordered by expert, then by t k + j.  Chosen
    // expert d (its rank among the chosen ones) counts its pairs per token;
    // its first pair is the sum of the counts of the experts below it, and
    // a pair's rank among its expert's pairs is that expert's count in the
    // tokens before t plus its earlier places in token t (a token lists an
    // expert twice only through given or replaced ids).  Each expert's
    // pairs are then cut into slots of at most 8 (the columns of one MMA).
    auto rank_of = [&](int e) { return wprefix[e >> 5] + __popc(bitmap[e >> 5] & ((1u << (e & 31)) - 1u)); };
    for (int i = tid; i < tk; i += kThreads) {
        const int e = ids_s[i], t = i / k, d = rank_of(e);
        atomicAdd(&tcount[2 * d + (t >> 2)], 1u << (8 * (t & 3)));
        dexp[d] = e;
    }
    __syncthreads();
    DEC_MARK(9);
    if (warp == 0) {
        const int nchosen = wprefix[32];
        int carry = 0;   // (pairs << 16) | slots of the experts so far
        for (int d0 = 0; d0 < nchosen; d0 += 32) {
            const int d = d0 + lane;
            int c = 0;
            if (d < nchosen) {
                const uint64_t v = (uint64_t)tcount[2 * d] | (uint64_t)tcount[2 * d + 1] << 32;
#pragma unroll
                for (int b = 0; b < kN; ++b)
                    c += (int)((v >> (8 * b)) & 0xFFu);
            }
            const int mine = (c << 16) | ((c + 7) >> 3);   // both sums stay below 2^16
            int incl = mine;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o)
                    incl += n;
            }
            if (d < nchosen) {
                const int excl = carry + incl - mine;
                const int base = excl >> 16, sl0 = excl & 0xFFFF, e = dexp[d];
                dbase[d] = base;
                for (int q = 0; 8 * q < c; ++q) {
                    slot_e[sl0 + q] = e;
                    slot_base[sl0 + q] = base + 8 * q;
                    slot_cnt[sl0 + q] = c - 8 * q < 8 ? c - 8 * q : 8;
                }
            }
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0)
            flag[2] = carry & 0xFFFF;   // routed slots
    }
    __syncthreads();
    DEC_MARK(10);
    const int nd_routed = flag[2];
    for (int i = tid; i < tk; i += kThreads) {
        const int e = ids_s[i], t = i / k, j = i % k, d = rank_of(e);
        const uint64_t v = (uint64_t)tcount[2 * d] | (uint64_t)tcount[2 * d + 1] << 32;
        int before = 0;
        for (int t2 = 0; t2 < t; ++t2)
            before += (int)((v >> (8 * t2)) & 0xFFu);
        for (int j2 = 0; j2 < j; ++j2)
            before += ids_s[t * k + j2] == e;
        const int p = dbase[d] + before;
        pair_tok[p] = t;
        pair_w[p] = w_s[i];
        pidx[i] = p;
    }
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

    // ------------------------------------------------ C: gate/up + SwiGLU (tensor cores)
    {
        const int gsh = WFMT == MOE_WFMT_Q4K ? 8 : gshift;
        const int cpg = chunks_per_group<WFMT>(A.G);
        const int per_slot = I / kFeat;
        const int U = Nd * per_slot;
        const int npass = (nchH + 4 * kWarps - 1) / (4 * kWarps);
        // this warp's items: (unit u, pass), units u = blockIdx.x + gridDim.x i
        const int nunits = U > (int)blockIdx.x ? (U - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
        const int nitems = nunits * npass;
        auto unit_of = [&](int it) { return (int)blockIdx.x + (int)gridDim.x * (it / npass); };
        auto stage = [&](int it2) {
            if (it2 < nitems) {
                const int u2 = unit_of(it2), pass2 = it2 % npass;
                gu_stage<WFMT>(A, slot_e[u2 / per_slot], (u2 % per_slot) * kFeat, pass2 * 4 * kWarps, nchH, gsh, warp,
                               lane, mybuf_s + (it2 % NS) * kIB);
            }
            cp_async_commit();
        };
        for (int it2 = 0; it2 < NS - 1; ++it2)
            stage(it2);
        float acc[2][4];
        int ru = 0;   // units reduced so far: picks the partials buffer
        DEC_DECL(ts);
        DEC_DECL(tw);
        DEC_DECL(tc);
        DEC_DECL(tr);
#ifdef MOEQ4_TRACE
        if (blockIdx.x < 4 && threadIdx.x == 0)
            g_dec_trace[blockIdx.x][16] = (unsigned long long)clock64();
#endif
        for (int it = 0; it < nitems; ++it) {
            const int u = unit_of(it), pass = it % npass;
            const int d = u / per_slot, f0 = (u % per_slot) * kFeat;
            const int base = slot_base[d], cnt = slot_cnt[d];
            DEC_CLK(c_s);
            stage(it + NS - 1);
            DEC_ACC(ts, c_s);
            if (pass == 0) {
#pragma unroll
                for (int m = 0; m < 2; ++m)
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        acc[m][v] = 0.f;
            }
            // this lane's B column: token gid of the unit's expert (zero row past cnt)
            const int trow = gid < cnt ? pair_tok[base + gid] : kN;
            const int tA = 2 * tid4 < cnt ? pair_tok[base + 2 * tid4] : -1;
            const int tB = 2 * tid4 + 1 < cnt ? pair_tok[base + 2 * tid4 + 1] : -1;
            DEC_CLK(c_w);
            cp_async_wait_upto(NS - 1);   // item it's copies have landed
            __syncwarp();
            DEC_ACC(tw, c_w);
            DEC_CLK(c_c);
            const uint8_t *buf = mybuf + (it % NS) * kIB;
            // the warp's 4 consecutive chunks (all past the end or none: H is
            // a multiple of 128); the MMAs of one scale group accumulate in
            // dd and the group's scale and offset are applied once
            const int j0 = pass * 4 * kWarps + 4 * warp;
            if (j0 < nchH) {
                float dd[2][4] = {};
                float sA = 0.f, sB = 0.f;
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    const int j = j0 + n;
                    sA += tA >= 0 ? xsum[tA * nchH + j] : 0.f;
                    sB += tB >= 0 ? xsum[tB * nchH + j] : 0.f;
                    const uint16_t *brow = xb + (size_t)trow * XS + j * 32;
#pragma unroll
                    for (int m = 0; m < 2; ++m) {
                        const uint4 lo = *(const uint4 *)(buf + ((n * 2 + m) * 16 + gid) * 16);
                        const uint4 hi = *(const uint4 *)(buf + ((n * 2 + m) * 16 + gid + 8) * 16);
                        chunk_mma(dd[m], lo, hi, brow, tid4);
                    }
                    if (((n + 1) & (cpg - 1)) == 0) {   // the last chunk of a scale group
                        // rows gid (v = 0, 1) and gid + 8 (v = 2, 3); tokens 2 tid4 + (v & 1)
#pragma unroll
                        for (int m = 0; m < 2; ++m) {
                            const uint8_t *mrow = buf + kCodeBuf + ((n * 2 + m) * 16 + gid) * kMB;
                            float alo, blo, ahi, bhi;
                            staged_coeffs<WFMT>(mrow, j * 32, alo, blo);
                            staged_coeffs<WFMT>(mrow + 8 * kMB, j * 32, ahi, bhi);
#pragma unroll
                            for (int v = 0; v < 4; ++v) {
                                const float sx = (v & 1) ? sB : sA;
                                const float a = (v >> 1) ? ahi : alo, b = (v >> 1) ? bhi : blo;
                                acc[m][v] = fmaf(a, fmaf(-kOff, sx, dd[m][v]), fmaf(b, sx, acc[m][v]));
                                dd[m][v] = 0.f;
                            }
                        }
                        sA = 0.f;
                        sB = 0.f;
                    }
                }
            }
            __syncwarp();
            DEC_ACC(tc, c_c);
            DEC_CLK(c_r);
            if (pass == npass - 1) {
                // the unit is complete in every warp: gate and up summed over
                // the warps, in order.  The partials alternate between two
                // buffers: a buffer is written again two units later, after a
                // block barrier that its readers pass only once they are done,
                // so one barrier per unit suffices and the other warps go on
                // to the next unit while the sums are formed.
                float *rb = red + (size_t)(ru & (L.nred - 1)) * kWarps * 2 * L.ntok * kRedLd;
                ++ru;
                if (L.nred == 1)
                    __syncthreads();   // the previous unit's sums are formed
#pragma unroll
                for (int m = 0; m < 2; ++m)
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const int nn = 2 * tid4 + (v & 1);
                        if (nn < cnt)
                            rb[((warp * 2 + m) * L.ntok + nn) * kRedLd + gid + 8 * (v >> 1)] = acc[m][v];
                    }
                __syncthreads();
                if (tid < kFeat * cnt) {
                    const int nn = tid / kFeat, f = tid % kFeat;
                    float g = 0.f, uu = 0.f;
                    for (int w = 0; w < kWarps; ++w) {
                        g += rb[((w * 2 + 0) * L.ntok + nn) * kRedLd + f];
                        uu += rb[((w * 2 + 1) * L.ntok + nn) * kRedLd + f];
                    }
                    const float hv = g / (1.0f + expf(-g)) * uu;
                    A.h[(size_t)(base + nn) * I + f0 + f] = (uint16_t)(pack_bf16x2(hv, 0.f) & 0xFFFFu);
                }
            }
            DEC_ACC(tr, c_r);
        }
        cp_async_wait_group<0>();
        __syncwarp();
#ifdef MOEQ4_TRACE
        if (blockIdx.x < 4 && threadIdx.x == 0) {
            g_dec_trace[blockIdx.x][11] = (unsigned long long)ts;
            g_dec_trace[blockIdx.x][12] = (unsigned long long)tw;
            g_dec_trace[blockIdx.x][13] = (unsigned long long)tc;
            g_dec_trace[blockIdx.x][14] = (unsigned long long)tr;
            g_dec_trace[blockIdx.x][17] = (unsigned long long)clock64();
        }
#endif
    }
    DEC_MARK(4);
    if (!grid_sync(A.bar, A.status, 92, flag, false, wait_ns))
        return;
    DEC_MARK(5);

    // ------------------------------------------------ D: down + combine (tensor cores)
    {
        // h as bf16 rows of I + 8 elements (row NP is zeros) and fp32 chunk sums
        const int HS = I + 8;
        uint16_t *hb = (uint16_t *)(smem + L.big);
        float *hsum = (float *)(hb + (size_t)(NP + 1) * HS);
        issue_rows(A.h, I, NP, NP, smem_u32(hb), HS, tid);
        const int gsh = WFMT == MOE_WFMT_Q4K ? 8 : gshift;
        const int cpg = chunks_per_group<WFMT>(A.G);
        const int nparts = (nchI + 7) / 8;
        float *o_s = (float *)(smem + L.ored);   // [pair][column]
        // this warp's slots: d = warp + kWarps i; items (slot, part)
        const int nslots = Nd > warp ? (Nd - 1 - warp) / kWarps + 1 : 0;
        const int nitems = nslots * nparts;
        auto stage_for = [&](int c0, int it2) {
            if (it2 < nitems)
                dn_stage<WFMT>(A, slot_e[warp + kWarps * (it2 / nparts)], c0, it2 % nparts, nchI, gsh, lane,
                               mybuf_s + (it2 % NS) * kIB);
            cp_async_commit();
        };
        // the first column block's weights are requested before h is waited for
        const int c_first = (int)blockIdx.x * kCols;
        for (int it2 = 0; it2 < NS - 1; ++it2)
            stage_for(c_first < H ? c_first : 0, c_first < H ? it2 : nitems);
        cp_async_wait_upto(NS - 1);   // h (the oldest group) has landed
        __syncthreads();
        row_sums(hb, I, NP, HS, hsum, tid);
        __syncthreads();
        DEC_DECL(tdw);
        for (int u = blockIdx.x; u < H / kCols; u += gridDim.x) {
            const int c0 = u * kCols;
            auto stage = [&](int it2) { stage_for(c0, it2); };
            if (u != (int)blockIdx.x)
                for (int it2 = 0; it2 < NS - 1; ++it2)
                    stage(it2);
            float acc[4];
            for (int it = 0; it < nitems; ++it) {
                const int d = warp + kWarps * (it / nparts), q = it % nparts;
                const int base = slot_base[d], cnt = slot_cnt[d];
                stage(it + NS - 1);
                if (q == 0) {
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        acc[v] = 0.f;
                }
                const int prow = gid < cnt ? base + gid : NP;
                const int pA = 2 * tid4 < cnt ? base + 2 * tid4 : -1;
                const int pB = 2 * tid4 + 1 < cnt ? base + 2 * tid4 + 1 : -1;
                DEC_CLK(c0);
                cp_async_wait_upto(NS - 1);
                __syncwarp();
                DEC_ACC(tdw, c0);
                const uint8_t *buf = mybuf + (it % NS) * kIB;
                // the item's chunks (past the end in whole groups of 4: I is a
                // multiple of 128); the MMAs of one scale group accumulate in
                // dd and the group's scale and offset are applied once
                float dd[4] = {0.f, 0.f, 0.f, 0.f};
                float sA = 0.f, sB = 0.f;
#pragma unroll 4
                for (int n = 0; n < 8; ++n) {
                    const int j = 8 * q + n;
                    if (j < nchI) {
                        sA += pA >= 0 ? hsum[pA * nchI + j] : 0.f;
                        sB += pB >= 0 ? hsum[pB * nchI + j] : 0.f;
                        const uint4 lo = *(const uint4 *)(buf + (n * 16 + gid) * 16);
                        const uint4 hi = *(const uint4 *)(buf + (n * 16 + gid + 8) * 16);
                        chunk_mma(dd, lo, hi, hb + (size_t)prow * HS + j * 32, tid4);
                        if (((n + 1) & (cpg - 1)) == 0) {   // the last chunk of a scale group
                            float clo_a, clo_b, chi_a, chi_b;
                            const uint8_t *mrow = buf + kCodeBuf + (n * 16 + gid) * kMB;
                            staged_coeffs<WFMT>(mrow, j * 32, clo_a, clo_b);
                            staged_coeffs<WFMT>(mrow + 8 * kMB, j * 32, chi_a, chi_b);
#pragma unroll
                            for (int v = 0; v < 4; ++v) {
                                const float sx = (v & 1) ? sB : sA;
                                const float a = (v >> 1) ? chi_a : clo_a, b = (v >> 1) ? chi_b : clo_b;
                                acc[v] = fmaf(a, fmaf(-kOff, sx, dd[v]), fmaf(b, sx, acc[v]));
                                dd[v] = 0.f;
                            }
                            sA = 0.f;
                            sB = 0.f;
                        }
                    }
                }
                __syncwarp();
                if (q == nparts - 1) {
                    // o[pair][column] for the slot's pairs: rows gid, gid + 8 are columns of y
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const int nn = 2 * tid4 + (v & 1);
                        if (nn < cnt)
                            o_s[(base + nn) * kRedLd + gid + 8 * (v >> 1)] = acc[v];
                    }
                }
            }
            cp_async_wait_group<0>();
            __syncthreads();
            // the combine of these columns: routed experts in j order, then the shared expert
            if (tid < T * kCols) {
                const int t = tid / kCols, c2 = tid % kCols;
                float y = 0.f;
                for (int jj = 0; jj < k; ++jj)
                    y = fmaf(w_s[t * k + jj], o_s[pidx[t * k + jj] * kRedLd + c2], y);
                if (A.has_shared)
                    y = fmaf(w_s[tk + t], o_s[(tk + t) * kRedLd + c2], y);
                A.y[(size_t)t * H + c0 + c2] = (uint16_t)(pack_bf16x2(y, 0.f) & 0xFFFFu);
            }
            __syncthreads();
        }
#ifdef MOEQ4_TRACE
        if (blockIdx.x < 4 && threadIdx.x == 0)
            g_dec_trace[blockIdx.x][15] = (unsigned long long)tdw;
#endif
    }
    DEC_MARK(6);
}

}  // namespace

cudaError_t launch_decode_layer(const DecodeArgs &a, int grid, cudaStream_t st)
{
    const DecodeSmem L = decode_smem_layout(a.T, a.k, a.H, a.I, a.has_shared, a.wfmt);
    void (*kern)(const DecodeArgs, const DecodeSmem) =
        a.wfmt == MOE_WFMT_Q4K             ? decode_layer_kernel<MOE_WFMT_Q4K>
        : a.wfmt == MOE_WFMT_INT4_ASYM     ? decode_layer_kernel<MOE_WFMT_INT4_ASYM>
        : a.wfmt == MOE_WFMT_INT4_SYM_F16 ? decode_layer_kernel<MOE_WFMT_INT4_SYM_F16>
                                           : decode_layer_kernel<MOE_WFMT_INT4_SYM>;
    // the opt-in limit once per device and format (callers never ask for
    // more: see the admission check)
    static std::atomic<bool> configured[64][4];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    const int f = a.wfmt >= 0 && a.wfmt < 4 ? a.wfmt : 0;
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
