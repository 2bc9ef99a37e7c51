// Grouped expert GEMMs on 4-bit weights (and the router GEMM), tcgen05 tensor cores.
//
// hipfire 0.4.3 benchmarks, "Read this before comparing columns": the MoE
// prefill route either keeps per-expert buffers or takes the "symmetric
// IU4 MoE" route for int4 symmetric experts.  This kernel is the B200
// counterpart of that route: the rows of the token permutation are cut into
// tiles per expert, and each tile runs
//     D[feature, token] = sum_K  W[feature, K] * X[token, K]
// with the weights as the MMA's M = 128 side.  Blackwell has no 4-bit
// operand for kind::f16 MMAs, so the codes are expanded to bf16 on chip:
// dequant warps write them straight into tensor memory (TMEM), where the
// MMA reads its A operand, and the tokens are gathered into swizzled
// shared memory as the B operand.  The accumulator stays in TMEM until the
// epilogue warps apply SwiGLU (gate/up pass), round to bf16 (down pass) or
// add the router bias (router pass).
//
// The router pass uses the same engine: its fp32 weights are split into two
// bf16 parts (hi + lo carry 16 significand bits, the rest is below the fp32
// accumulation error of the tensor cores over K = 2048), both products are
// exact in fp32 and accumulate into one fp32 accumulator.
//
// Warp roles of one persistent CTA (one per SM, 768 threads):
//   warp 0      gathers token rows of B with cp.async (zero rows past the tail)
//   warp 1      issues tcgen05.mma (one thread) and commits stage releases
//   warp 2      streams code blocks and per-tile scale blocks with bulk copies
//   warp 3      owns the TMEM allocation; in the router pass it also forms
//               the shared expert's gate logits x . g
//   warps 4-19  dequantise, in two groups of eight taking alternate k-steps:
//               row r = 32*(warp%4) + lane, half c of the k-step = ((warp-4)%8)/4
//   warps 20-23 epilogue (TMEM -> registers -> global)
// Every wait is bounded; on timeout the CTA records MOE_ERR_TIMEOUT and
// unwinds.
#include <cstdint>
#include <cuda_runtime.h>

#include "dequant.cuh"
#include "kernels.h"
#include "moeq4.h"
#include "ptx.cuh"

namespace moeq4 {

// Optional timeline instrumentation: with -DMOEQ4_TRACE the first four CTAs
// record %globaltimer at pipeline events into g_trace[cta][event][step]
// (read back with moe_trace_fetch); without it the hooks compile to nothing.
#if defined(MOEQ4_TRACE) && defined(MOEQ4_TRACE_WARPS)
#define TRACE_OTHER(ev, step) do { } while (0)
#else
#define TRACE_OTHER(ev, step) TRACE_EVENT(ev, step)
#endif
#ifdef MOEQ4_TRACE
constexpr int kTraceSteps = 512;
__device__ unsigned long long g_trace[4][16][kTraceSteps];
#define TRACE_EVENT(ev, step)                                                          \
    do {                                                                               \
        if (blockIdx.x < 4 && (step) >= 0 && (step) < kTraceSteps)                     \
            g_trace[blockIdx.x][(ev)][(step)] = globaltimer_ns();                      \
    } while (0)
#else
#define TRACE_EVENT(ev, step) \
    do {                      \
    } while (0)
#endif

constexpr int kBNMax = 128;  // max tokens per tile (the MMA's N); tiles of 64 when groups are small
constexpr int kStages = 4;   // B / TMEM-A pipeline depth
constexpr int kEpiTok = 16;  // tokens per epilogue chunk
constexpr int kEpiStride = 80;                                   // bytes per staged token row (64 + pad)
constexpr int kEpiBytes = 4 * kEpiTok * kEpiStride;              // staging for the four epilogue warps
constexpr int kDeqGroups = 2;                  // dequant warp groups, alternating k-steps
constexpr int kThreads = (8 + 8 * kDeqGroups) * 32;

enum { MODE_GATE_UP = 0, MODE_DOWN = 1, MODE_ROUTER = 2 };

template <int MODE, int BN>
struct Geo {
    static constexpr int kBN = BN;
    static constexpr int kNA = MODE == MODE_DOWN ? 1 : 2;                               // A operands per k-step
    static constexpr int kNAcc = MODE == MODE_GATE_UP ? 2 : 1;                          // accumulators per unit
    static constexpr int kNAcc_ = MODE == MODE_GATE_UP ? 2 : 1;
    // as many accumulator buffers (up to 2) as TMEM holds next to the A stages:
    // with two, the epilogue of one tile overlaps the MMAs of the next
    static constexpr int kAccBufs = (512 - kStages * kNA * 32) / (kNAcc_ * BN) >= 2 ? 2 : 1;
    static constexpr int kNCode = MODE == MODE_GATE_UP ? 2 : MODE == MODE_DOWN ? 1 : 0; // code matrices
    static constexpr int kCodeStages = MODE == MODE_GATE_UP ? 8 : MODE == MODE_DOWN ? 16 : 1;
    static constexpr int kCodeBytes = kCodeStages * (kNCode ? code_block_bytes(kNCode) : 0);
    static constexpr int kBBytes = kStages * BN * 128;
    static constexpr int kAccCols = kAccBufs * kNAcc * BN;
    static constexpr int kTmemCols = 512;
    static_assert(kAccCols + kStages * kNA * 32 <= kTmemCols, "TMEM budget");
    static constexpr bool kGather = MODE == MODE_GATE_UP;
};

struct Barriers {
    uint64_t full[kStages];       // A dequantised into TMEM and B gathered into shared memory
    uint64_t mma_done[kStages];
    uint64_t code_full[16];
    uint64_t code_empty[16];
    uint64_t meta_full[2];
    uint64_t meta_empty[2];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int never_abort;   // stays 0: a wait that must not be cut short by an abort
};

struct Unit {
    int e, f, row0, nvalid, nmma;
};

struct Sched {
    const int *tile_start;   // [E_total + 1] first tile of each expert
    const int *row_start;    // [E_total] first permuted row
    const int *row_count;    // [E_total] rows
};

template <int BN>
__device__ __forceinline__ Unit decode_unit(int u, const GemmArgs &p, const Sched &sc)
{
    Unit r;
    const int tile = u / p.F;
    r.f = u - tile * p.F;
    int lo = 0, hi = p.E_total - 1;   // largest e with tile_start[e] <= tile (a non-empty expert)
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sc.tile_start[mid] <= tile)
            lo = mid;
        else
            hi = mid - 1;
    }
    r.e = lo;
    const int c = tile - sc.tile_start[lo];
    r.row0 = sc.row_start[lo] + c * BN;
    r.nvalid = min(BN, sc.row_count[lo] - c * BN);
    r.nmma = max(16, (r.nvalid + 15) & ~15);
    return r;
}

// Every CTA derives the tile schedule from the permutation offsets: rows of
// expert e are [offsets[e], offsets[e+1]); the shared expert (if any) is
// expert E with rows [T k, T k + T); expert e owns ceil(rows / BN) tiles.
// Without offsets (router pass) the T token rows form a single group.
template <int BN>
__device__ void build_schedule(const GemmArgs &p, int *s_tile_start, int *s_row_start, int *s_row_count,
                               int *s_part)
{
    const int n = p.E_total;
    const int per = (n + kThreads - 1) / kThreads;
    const int e0 = threadIdx.x * per;
    int local = 0;
    for (int e = e0; e < min(n, e0 + per); ++e) {
        int start, cnt;
        if (!p.offsets) {
            start = 0;
            cnt = p.T;
        } else if (e < p.E) {
            start = p.offsets[e];
            cnt = p.offsets[e + 1] - p.offsets[e];
        } else {
            start = p.Tk;
            cnt = p.T;
        }
        s_row_start[e] = start;
        s_row_count[e] = cnt;
        local += (cnt + BN - 1) / BN;
    }
    s_part[threadIdx.x] = local;
    __syncthreads();
    for (int off = 1; off < kThreads; off <<= 1) {
        const int v = threadIdx.x >= off ? s_part[threadIdx.x - off] : 0;
        __syncthreads();
        s_part[threadIdx.x] += v;
        __syncthreads();
    }
    int run = s_part[threadIdx.x] - local;
    for (int e = e0; e < min(n, e0 + per); ++e) {
        s_tile_start[e] = run;
        run += (s_row_count[e] + BN - 1) / BN;
    }
    if (threadIdx.x == kThreads - 1)
        s_tile_start[n] = s_part[kThreads - 1];
}

// fp32 -> two bf16 parts (hi, lo): w - hi is exact in fp32, so hi + lo
// matches w to about 2^-17 relative.
__device__ __forceinline__ void split2(float w0, float w1, uint32_t &hi, uint32_t &lo)
{
    hi = pack_bf16x2(w0, w1);
    const float r0 = w0 - __uint_as_float(hi << 16);
    const float r1 = w1 - __uint_as_float(hi & 0xFFFF0000u);
    lo = pack_bf16x2(r0, r1);
}

template <int MODE, int WFMT, int BN>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_kernel(const GemmArgs p)
{
    using L = Geo<MODE, BN>;
    constexpr int kBN = BN;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the swizzled B stages
    // offset arithmetic on the shared array keeps the pointer in the shared
    // window (a round trip through an integer would make every access generic)
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *sB = smem;
    uint8_t *sCode = sB + L::kBBytes;
    uint8_t *sMeta = sCode + L::kCodeBytes;
    const int meta_bytes = p.meta_bytes;
    const int meta_al = (meta_bytes + 127) & ~127;
    Barriers *bars = (Barriers *)(sMeta + 2 * meta_al);
    int *s_tile_start = (int *)(bars + 1);
    int *s_row_start = s_tile_start + p.E_total + 1;
    int *s_row_count = s_row_start + p.E_total;
    int *s_part = s_row_count + p.E_total;
    uint8_t *s_epi = (uint8_t *)(s_part + kThreads);
    s_epi += (16u - (smem_u32(s_epi) & 15u)) & 15u;    // epilogue staging, 16-byte aligned
    const Sched sched{s_tile_start, s_row_start, s_row_count};

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            // eight dequant warps + one cp.async completion arrival per lane of the B producer
            mbar_init(&bars->full[s], 8 + 32);
            mbar_init(&bars->mma_done[s], 1);
        }
        for (int s = 0; s < L::kCodeStages; ++s) {
            mbar_init(&bars->code_full[s], 1);
            mbar_init(&bars->code_empty[s], 8);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->meta_full[s], 1);
            mbar_init(&bars->meta_empty[s], 8 * kDeqGroups);
            mbar_init(&bars->acc_full[s], 1);
            mbar_init(&bars->acc_empty[s], 4);
        }
        mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        bars->never_abort = 0;
        fence_mbar_init();
    }
    build_schedule<BN>(p, s_tile_start, s_row_start, s_row_count, s_part);
    if (warp == 3) {
        tmem_alloc(&bars->tmem_base, L::kTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    const int total_units = s_tile_start[p.E_total] * p.F;
    const int KS = p.K / kKStep;
    WaitCtx wc{&bars->abort_flag, p.status, globaltimer_ns()};

    if (warp == 0) {
        // ------------------------------------------------ B producer (gather)
        int step = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
            const Unit un = decode_unit<BN>(u, p, sched);
            const uint16_t *src[kBN / 32];
            uint32_t bytes[kBN / 32];
#pragma unroll
            for (int i = 0; i < kBN / 32; ++i) {
                const int r = lane + 32 * i;
                const int prow = un.row0 + r;
                int srow = 0;
                if (r < un.nvalid)
                    srow = L::kGather ? (prow < p.Tk ? p.sorted_slot[prow] / p.topk : prow - p.Tk) : prow;
                src[i] = p.b_src + (size_t)srow * p.ldb;
                bytes[i] = r < un.nvalid ? 16u : 0u;
            }
            for (int ks = 0; ks < KS; ++ks, ++step) {
                const int s = step % kStages;
                if (step >= kStages && !mbar_wait(&bars->mma_done[s], ((step / kStages) & 1) ^ 1, wc, 1)) {
                    ok = false;
                    break;
                }
                const uint32_t base = smem_u32(sB + s * kBN * 128);
#pragma unroll
                for (int i = 0; i < kBN / 32; ++i) {
                    const int r = lane + 32 * i;
                    if (r < un.nmma) {
                        const uint32_t rbase = base + (r >> 3) * 1024 + (r & 7) * 128;
                        const uint16_t *g = src[i] + ks * kKStep;
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            cp_async_16(rbase + ((j ^ (r & 7)) << 4), g + j * 8, bytes[i]);
                    }
                }
                // this lane's copies for the stage arrive on full[s] when they land
                cp_async_arrive_noinc(&bars->full[s]);
                if (lane == 0)
                    TRACE_OTHER(0, step);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (converged warp, one elected lane)
        int step = 0, uidx = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++uidx) {
            const Unit un = decode_unit<BN>(u, p, sched);
            const uint32_t idesc = idesc_bf16_f32(128, un.nmma);
            const int ab = uidx % L::kAccBufs;
            const uint32_t acc = tmem + ab * L::kNAcc * kBN;
            if (uidx >= L::kAccBufs) {
                if (!mbar_wait(&bars->acc_empty[ab], ((uidx / L::kAccBufs) & 1) ^ 1, wc, 2))
                    break;
                tc_fence_after();
            }
            for (int ks = 0; ks < KS; ++ks, ++step) {
                const int s = step % kStages;
                const uint32_t ph = (step / kStages) & 1;
                // every lane polls the same barrier, so the outcome is warp-uniform
                if (!mbar_wait(&bars->full[s], ph, wc, 3)) {
                    ok = false;
                    break;
                }
                if (lane == 0)
                    TRACE_OTHER(9, step);
                // the B stage was written by cp.async (generic proxy); the MMA
                // reads it through the async proxy
                fence_proxy_async_smem();
                tc_fence_after();
                const uint64_t bdesc0 = sdesc_kmajor_sw128(smem_u32(sB + s * kBN * 128));
                const uint32_t a_base = tmem + L::kAccCols + s * L::kNA * 32;
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bdesc = bdesc0 + (uint64_t)(kk * 2);   // +32 bytes along K
#pragma unroll
                        for (int m = 0; m < L::kNA; ++m) {
                            const uint32_t a_t = a_base + m * 32 + kk * 8;
                            if (MODE == MODE_ROUTER)   // both parts into one accumulator
                                mma_ts_f16(acc, a_t, bdesc, idesc, (ks | kk | m) != 0);
                            else
                                mma_ts_f16(acc + m * kBN, a_t, bdesc, idesc, (ks | kk) != 0);
                        }
                    }
                    mma_commit(&bars->mma_done[s]);
                }
                __syncwarp();
                if (lane == 0)
                    TRACE_OTHER(5, step);
            }
            if (ok) {
                if (elect_one())
                    mma_commit(&bars->acc_full[ab]);
                __syncwarp();
            }
        }
        // all issued MMAs finish before the CTA may release TMEM
        if (elect_one())
            mma_commit(&bars->drain);
        __syncwarp();
        WaitCtx wd{&bars->never_abort, p.status, globaltimer_ns()};   // drain even after an abort
        warp_wait(&bars->drain, 0, wd, 5);
    } else if (warp == 2) {
        // ------------------------------------------------ code / meta producer (converged warp)
        if (MODE != MODE_ROUTER) {
            int step = 0, munit = 0;
            const int cbytes = code_block_bytes(L::kNCode);
            bool ok = true;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++munit) {
                const Unit un = decode_unit<BN>(u, p, sched);
                const size_t tile_id = (size_t)un.e * p.F + un.f;
                const int mb = munit & 1;
                if (munit >= 2 && !warp_wait(&bars->meta_empty[mb], ((munit >> 1) & 1) ^ 1, wc, 6))
                    break;
                if (elect_one()) {
                    mbar_arrive_expect_tx(&bars->meta_full[mb], meta_bytes);
                    bulk_g2s(sMeta + mb * meta_al, p.wmeta + tile_id * meta_bytes, meta_bytes, &bars->meta_full[mb]);
                }
                __syncwarp();
                for (int ks = 0; ks < KS; ++ks, ++step) {
                    const int s = step % L::kCodeStages;
                    if (step >= L::kCodeStages &&
                        !warp_wait(&bars->code_empty[s], ((step / L::kCodeStages) & 1) ^ 1, wc, 7)) {
                        ok = false;
                        break;
                    }
                    if (elect_one()) {
                        mbar_arrive_expect_tx(&bars->code_full[s], cbytes);
                        bulk_g2s(sCode + s * cbytes, p.wq + (tile_id * KS + ks) * cbytes, cbytes,
                                 &bars->code_full[s]);
                    }
                    __syncwarp();
                    if (lane == 0)
                        TRACE_OTHER(1, step);
                }
            }
        }
    } else if (warp == 3) {
        // ------------------------------------------------ shared-expert gate logits
        if (MODE == MODE_ROUTER && p.gate_w) {
            for (int t = blockIdx.x; t < p.T; t += gridDim.x) {
                const uint16_t *xr = p.b_src + (size_t)t * p.ldb;
                float acc = 0.f;
                for (int c0 = lane * 8; c0 < p.K; c0 += 256) {
                    const uint4 v = *(const uint4 *)(xr + c0);
                    const float4 g0 = *(const float4 *)(p.gate_w + c0);
                    const float4 g1 = *(const float4 *)(p.gate_w + c0 + 4);
                    acc = fmaf(__uint_as_float(v.x << 16), g0.x, acc);
                    acc = fmaf(__uint_as_float(v.x & 0xFFFF0000u), g0.y, acc);
                    acc = fmaf(__uint_as_float(v.y << 16), g0.z, acc);
                    acc = fmaf(__uint_as_float(v.y & 0xFFFF0000u), g0.w, acc);
                    acc = fmaf(__uint_as_float(v.z << 16), g1.x, acc);
                    acc = fmaf(__uint_as_float(v.z & 0xFFFF0000u), g1.y, acc);
                    acc = fmaf(__uint_as_float(v.w << 16), g1.z, acc);
                    acc = fmaf(__uint_as_float(v.w & 0xFFFF0000u), g1.w, acc);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
                    acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
                if (lane == 0)
                    p.gate_out[t] = acc;
            }
        }
    } else if (warp >= 4 && warp < 4 + 8 * kDeqGroups) {
        // ------------------------------------------------ dequant into TMEM
        const int dw = warp - 4;
        const int grp = dw / 8;                   // this group handles k-steps with step % kDeqGroups == grp
        const int c = (dw & 7) >> 2;              // which 32-element half of the k-step
        const int r = (warp & 3) * 32 + lane;     // tile row == TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        int step = 0, munit = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++munit) {
            const int mb = munit & 1;
            const uint8_t *meta = sMeta + mb * meta_al;
            float4 pre[8];                        // router: this row's next k-step, prefetched
            const float *wrow = nullptr;
            if (MODE == MODE_ROUTER) {
                const Unit un = decode_unit<BN>(u, p, sched);
                const int e = un.f * kTileRows + r;
                wrow = e < p.E ? p.a_f32 + (size_t)e * p.K + c * 32 : nullptr;
                const int ks0 = ((grp - step) % kDeqGroups + kDeqGroups) % kDeqGroups;   // first k-step of this group
                if (ks0 >= KS)
                    wrow = nullptr;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    pre[i] = wrow ? *(const float4 *)(wrow + ks0 * kKStep + 4 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
            } else if (!mbar_wait(&bars->meta_full[mb], (munit >> 1) & 1, wc, 8)) {
                break;
            }
            const int ngroups = WFMT == MOE_WFMT_Q4K ? p.K / 256 : p.K / max(p.G, 1);
            for (int ks = 0; ks < KS; ++ks, ++step) {
                if (step % kDeqGroups != grp)
                    continue;
                uint32_t words[L::kNA][16];
                if (MODE == MODE_ROUTER) {
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        v[4 * i] = pre[i].x;
                        v[4 * i + 1] = pre[i].y;
                        v[4 * i + 2] = pre[i].z;
                        v[4 * i + 3] = pre[i].w;
                    }
                    if (wrow && ks + kDeqGroups < KS) {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            pre[i] = *(const float4 *)(wrow + (ks + kDeqGroups) * kKStep + 4 * i);
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        split2(v[2 * j], v[2 * j + 1], words[0][j], words[1 % L::kNA][j]);
                } else {
                    const int sc = step % L::kCodeStages;
                    if (!mbar_wait(&bars->code_full[sc], (step / L::kCodeStages) & 1, wc, 9)) {
                        ok = false;
                        break;
                    }
#ifdef MOEQ4_TRACE_WARPS
                    if (lane == 0)
                        TRACE_EVENT((warp - 4) * 2, step);
#else
                    if (lane == 0 && warp == 4)
                        TRACE_EVENT(2, step);
#endif
                    const int kpos = ks * kKStep + c * 32;
                    const int cbytes = code_block_bytes(L::kNCode);
#pragma unroll
                    for (int m = 0; m < L::kNA; ++m) {
                        const uint4 codes =
                            lds128(smem_u32(sCode) + sc * cbytes + ((m * 2 + c) * kTileRows + r) * kChunkBytes);
                        if (WFMT == MOE_WFMT_Q4K) {
                            const int g = kpos / 256;
                            const uint4 hdr = lds128(smem_u32(meta) + ((m * ngroups + g) * kTileRows + r) * 16);
                            float dsc, dm;
                            q4k_subblock_scale(hdr, (kpos % 256) / 32, dsc, dm);
                            dequant_q4k_chunk(codes, dsc, dm, words[m]);
                        } else {
                            const int g = kpos / p.G;
                            const uint16_t sbits = lds16(smem_u32(meta) + ((m * ngroups + g) * kTileRows + r) * 2);
                            dequant_int4sym_chunk(codes, sbits, words[m]);
                        }
                    }
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&bars->code_empty[sc]);
                }
                const int sa = step % kStages;
#ifdef MOEQ4_TRACE_WARPS
                if (lane == 0)
                    TRACE_EVENT((warp - 4) * 2 + 1, step);
#else
                if (lane == 0 && warp == 4)
                    TRACE_EVENT(11, step);
#endif
                if (step >= kStages && !mbar_wait(&bars->mma_done[sa], ((step / kStages) & 1) ^ 1, wc, 10)) {
                    ok = false;
                    break;
                }
                if (lane == 0 && warp == 4)
                    TRACE_OTHER(12, step);
                tc_fence_after();
#pragma unroll
                for (int m = 0; m < L::kNA; ++m)
                    tmem_st16(tmem + lane_off + L::kAccCols + (sa * L::kNA + m) * 32 + c * 16, words[m]);
                tmem_wait_st();
                if (lane == 0 && warp == 4)
                    TRACE_OTHER(13, step);
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars->full[sa]);
                if (lane == 0 && warp == 4)
                    TRACE_OTHER(3, step);
                if (lane == 0 && warp == 11)
                    TRACE_OTHER(4, step);
            }
            if (MODE != MODE_ROUTER) {
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars->meta_empty[mb]);
            }
        }
    } else {
        // ------------------------------------------------ epilogue (last four warps)
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        int uidx = 0;
        for (int u = blockIdx.x; u < total_units; u += gridDim.x, ++uidx) {
            const Unit un = decode_unit<BN>(u, p, sched);
            const int ab = uidx % L::kAccBufs;
            if (!mbar_wait(&bars->acc_full[ab], (uidx / L::kAccBufs) & 1, wc, 11))
                break;
            tc_fence_after();
            if (lane == 0 && warp == 4 + 8 * kDeqGroups)
                TRACE_OTHER(6, uidx);
            const uint32_t acc = tmem + lane_off + ab * L::kNAcc * kBN;
            const int col = un.f * kTileRows + r;
            const int q = warp & 3;
            uint8_t *stage = s_epi + q * kEpiTok * kEpiStride;
            bool released = false;
            for (int n0 = 0; n0 < un.nmma; n0 += kEpiTok) {
                uint32_t g[16], v[16];
                tmem_ld16(acc + n0, g);
                if (L::kNAcc == 2)
                    tmem_ld16(acc + kBN + n0, v);
                tmem_wait_ld();
                if (n0 + kEpiTok >= un.nmma) {
                    // every column is in registers: hand the accumulator back to the MMA
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&bars->acc_empty[ab]);
                    released = true;
                }
                if (MODE == MODE_ROUTER) {
                    if (col < p.E) {
                        const float b = p.bias ? p.bias[col] : 0.f;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int n = n0 + j;
                            if (n < un.nvalid)
                                p.out_f32[(size_t)(un.row0 + n) * p.E + col] = __uint_as_float(g[j]) + b;
                        }
                    }
                } else {
                    // this lane's feature for 16 tokens -> staging [token][feature] (bf16)
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float o;
                        if (MODE == MODE_GATE_UP) {
                            const float a = __uint_as_float(g[j]);
                            o = __fdividef(a, 1.0f + __expf(-a)) * __uint_as_float(v[j]);   // silu(a) * u
                        } else {
                            o = __uint_as_float(g[j]);
                        }
                        *(__nv_bfloat16 *)(stage + j * kEpiStride + lane * 2) = __float2bfloat16_rn(o);
                    }
                    __syncwarp();
                    // lane: token n0 + (lane & 15), 32-byte half (lane >> 4) of the warp's 64-byte row slice
                    const int t = lane & 15, hh = lane >> 4;
                    const int n = n0 + t;
                    if (n < un.nvalid) {
                        const int prow = un.row0 + n;
                        uint16_t *dst = prow < p.Tk ? p.out + (size_t)prow * p.ldo
                                                    : p.out_shared + (size_t)(prow - p.Tk) * p.ldo;
                        uint4 *d4 = (uint4 *)(dst + un.f * kTileRows + q * 32 + hh * 16);
                        const uint4 *s4 = (const uint4 *)(stage + t * kEpiStride + hh * 32);
                        d4[0] = s4[0];
                        d4[1] = s4[1];
                    }
                    __syncwarp();
                }
            }
            if (!released) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars->acc_empty[ab]);
            }
            if (lane == 0 && warp == 4 + 8 * kDeqGroups)
                TRACE_OTHER(7, uidx);
        }
    }

    __syncthreads();
    if (warp == 3) {
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
    }
}

template <int MODE, int BN>
static size_t gemm_smem_bytes(int meta_bytes, int E_total)
{
    using L = Geo<MODE, BN>;
    const size_t need = 1024 + L::kBBytes + L::kCodeBytes + 2 * ((meta_bytes + 127) & ~127) + sizeof(Barriers) +
                        sizeof(int) * (3 * E_total + 1 + kThreads) + 16 + kEpiBytes;
    // at least half of the SM's shared memory, so that one CTA (and one TMEM
    // allocation) runs per SM
    return need > 116 * 1024 ? need : 116 * 1024;
}

template <int MODE, int WFMT, int BN>
static cudaError_t launch_one(const GemmArgs &a, int num_sms, cudaStream_t st)
{
    auto kern = grouped_gemm_kernel<MODE, WFMT, BN>;
    const size_t smem = gemm_smem_bytes<MODE, BN>(a.meta_bytes, a.E_total);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    kern<<<num_sms, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

size_t gemm_smem_required(int nmat, int meta_bytes, int E_total)
{
    // the 128-token tile is the larger of the two configurations
    return nmat == 2 ? gemm_smem_bytes<MODE_GATE_UP, 128>(meta_bytes, E_total)
                     : gemm_smem_bytes<MODE_DOWN, 128>(meta_bytes, E_total);
}

int gemm_tile_tokens(int T, int E, int k) { return (long long)T * k <= 64LL * E ? 64 : 128; }

template <int MODE, int BN>
static cudaError_t launch_fmt(const GemmArgs &a, int wfmt, int num_sms, cudaStream_t st)
{
    return wfmt == MOE_WFMT_Q4K ? launch_one<MODE, MOE_WFMT_Q4K, BN>(a, num_sms, st)
                                : launch_one<MODE, MOE_WFMT_INT4_SYM, BN>(a, num_sms, st);
}

cudaError_t launch_grouped_gemm(const GemmArgs &a, int nmat, int wfmt, int tile_tokens, int num_sms, cudaStream_t st)
{
    if (nmat == 2)
        return tile_tokens == 64 ? launch_fmt<MODE_GATE_UP, 64>(a, wfmt, num_sms, st)
                                 : launch_fmt<MODE_GATE_UP, 128>(a, wfmt, num_sms, st);
    return tile_tokens == 64 ? launch_fmt<MODE_DOWN, 64>(a, wfmt, num_sms, st)
                             : launch_fmt<MODE_DOWN, 128>(a, wfmt, num_sms, st);
}

// Router logits on tensor cores: logits[t, e] = x[t] . Wr[e] (+ bias[e]),
// and gate_out[t] = x[t] . g when g is given.
cudaError_t launch_router_gemm(const uint16_t *x, int T, int H, const float *wr, const float *bias, int E,
                               const float *gate_w, float *logits, float *gate_out, int *status, int num_sms,
                               cudaStream_t st)
{
    if (T == 0)
        return cudaSuccess;
    GemmArgs a{};
    a.b_src = x;
    a.ldb = H;
    a.T = T;
    a.E = E;
    a.E_total = 1;
    a.K = H;
    a.F = (E + kTileRows - 1) / kTileRows;
    a.a_f32 = wr;
    a.bias = bias;
    a.gate_w = gate_w;
    a.gate_out = gate_out;
    a.out_f32 = logits;
    a.status = status;
    return launch_one<MODE_ROUTER, 0, 128>(a, num_sms, st);
}

}  // namespace moeq4

#ifdef MOEQ4_TRACE
extern "C" int moe_trace_fetch(unsigned long long *host)
{
    return (int)cudaMemcpyFromSymbol(host, moeq4::g_trace, sizeof(moeq4::g_trace));
}
extern "C" int moe_trace_clear()
{
    static unsigned long long zero[4 * 16 * moeq4::kTraceSteps];
    return (int)cudaMemcpyToSymbol(moeq4::g_trace, zero, sizeof(zero));
}
#endif
