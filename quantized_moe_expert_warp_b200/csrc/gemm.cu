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
// epilogue warps apply SwiGLU (gate/up pass) or round to bf16 (down pass).
//
// Warp roles of one persistent CTA (one per SM, 768 threads):
//   warp 0      loads the token rows of B with one tiled TMA copy per k-step:
//               rows of x in permuted order (gate/up, routed experts), of x
//               (shared expert) or of h (down)
//   warp 1      issues tcgen05.mma (one thread) and commits stage releases
//   warp 2      streams code blocks and per-tile scale blocks with bulk copies
//   warp 3      owns the TMEM allocation
//   warps 4-19  dequantise, in two groups of eight taking alternate k-steps:
//               row r = 32*(warp%4) + lane, half c of the k-step = ((warp-4)%8)/4
//   warps 20-23 epilogue (TMEM -> registers -> global)
// Every wait is bounded; on timeout the CTA records MOE_ERR_TIMEOUT and
// unwinds.
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#ifdef MOEQ4_TRACE
// per wait site, summed over warps: [0] waits that polled more than once, [1] failed polls
__device__ unsigned long long g_wait_stats[16][2];
// cycle accounting of the first CTAs: per warp, clock cycles by pipeline phase
__device__ unsigned long long g_cyc[4][24][12];
#define CYC_DECL                                   \
    unsigned long long cyc_[12] = {0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0}; \
    long long cyc_t_ = clock64();
#define CYC(b)                                     \
    do {                                           \
        const long long n_ = clock64();            \
        cyc_[(b)] += (unsigned long long)(n_ - cyc_t_); \
        cyc_t_ = n_;                               \
    } while (0)
#define CYC_FLUSH                                                       \
    do {                                                                \
        if (blockIdx.x < 4 && lane == 0)                                \
            for (int i_ = 0; i_ < 12; ++i_)                             \
                g_cyc[blockIdx.x][warp][i_] = cyc_[i_];                 \
    } while (0)
#else
#define CYC_DECL
#define CYC(b) \
    do {       \
    } while (0)
#define CYC_FLUSH \
    do {          \
    } while (0)
#endif

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
        if (blockIdx.x < 4 && (ev) >= 0 && (ev) < 16 && (step) >= 0 && (step) < kTraceSteps) \
            g_trace[blockIdx.x][(ev)][(step)] = globaltimer_ns();                      \
    } while (0)
#else
#define TRACE_EVENT(ev, step) \
    do {                      \
    } while (0)
#endif

constexpr int kMaxAStages = 8;   // TMEM A-operand ring depth (dequantised k-steps), upper bound
#ifndef MOEQ4_A_STAGES_GU
#define MOEQ4_A_STAGES_GU 4
#endif
#ifndef MOEQ4_A_STAGES_DN
#define MOEQ4_A_STAGES_DN 8
#endif
#ifndef MOEQ4_B_STAGES_64
#define MOEQ4_B_STAGES_64 8
#endif
#ifndef MOEQ4_B_STAGES_128
#define MOEQ4_B_STAGES_128 4
#endif
constexpr int kMaxCodeChunks = 8;   // code ring: chunks of several k-steps, one bulk copy each
constexpr int kMaxMetaBufs = 4;
constexpr int kEpiTok = 16;  // tokens per epilogue chunk
constexpr int kEpiStride = 80;                                   // bytes per staged token row (64 + pad)
constexpr int kEpiBytes = 4 * kEpiTok * kEpiStride;              // staging for the four epilogue warps
#ifndef MOEQ4_DEQ_WARPS
#define MOEQ4_DEQ_WARPS 16
#endif
constexpr int kDeqWarps = MOEQ4_DEQ_WARPS;     // dequant warps (warps 4 .. 3 + kDeqWarps), a multiple of 8
constexpr int kThreads = (8 + kDeqWarps) * 32;

enum { MODE_GATE_UP = 0, MODE_DOWN = 1 };

template <int MODE, int BN>
struct Geo {
    static constexpr int kBN = BN;
    static constexpr int kNA = MODE == MODE_DOWN ? 1 : 2;                               // A operands per k-step
    static constexpr int kNAcc = MODE == MODE_GATE_UP ? 2 : 1;                          // accumulators per unit
    static constexpr int kNAcc_ = MODE == MODE_GATE_UP ? 2 : 1;
    // TMEM (512 columns): A stages of kNA x 32 columns, then as many
    // accumulator buffers (up to 2) as fit; with two, the epilogue of one
    // tile overlaps the MMAs of the next.  The requested A-stage count is cut
    // to leave room for one accumulator buffer.
    static constexpr int kAStagesReq = MODE == MODE_GATE_UP ? MOEQ4_A_STAGES_GU : MOEQ4_A_STAGES_DN;
    static constexpr int kAStagesFit = (512 - kNAcc_ * BN) / (kNA * 32);
    static constexpr int kAStages = kAStagesReq < kAStagesFit ? kAStagesReq : kAStagesFit;
    static_assert(kAStages >= 2 && kAStages <= kMaxAStages, "TMEM A stages");
    static constexpr int kAccBufs = (512 - kAStages * kNA * 32) / (kNAcc_ * BN) >= 2 ? 2 : 1;
    static constexpr int kNCode = MODE == MODE_GATE_UP ? 2 : 1;   // code matrices
    // dequant warp groups: groups of four warps, each warp a full k-step of
    // its 32 rows, or groups of eight, each warp one half of a k-step (any
    // warp count that would give more groups than TMEM A stages: a group must
    // not reuse a stage whose previous MMAs it has not waited for, so that no
    // mbarrier waiter runs two phases ahead)
    static constexpr int kGroupWarps = kDeqWarps / 4 > kAStages ? 8 : 4;
    static constexpr int kGroups = kDeqWarps / kGroupWarps;
    static_assert(kGroups <= kAStages, "dequant groups must not outnumber the TMEM A stages");
    static constexpr int kHalves = kGroupWarps == 8 ? 1 : 2;
    static constexpr int kCodeBlock = code_block_bytes(kNCode);
    // the gathered token rows wait on L2 / HBM latency, so their shared-memory
    // ring is deeper than the TMEM ring
    static constexpr int kBStages = BN == 64 ? MOEQ4_B_STAGES_64 : BN == 128 ? MOEQ4_B_STAGES_128 : 4;
    static_assert(kBStages <= 8, "B stages");
    // 256-token tiles only for the down pass: one accumulator of 256 columns
    // leaves room for eight A stages
    static_assert(BN != 256 || MODE == MODE_DOWN, "256-token tiles: down pass only");
    static constexpr int kBBytes = kBStages * BN * 128;
    static constexpr int kAccCols = kAccBufs * kNAcc * BN;
    static constexpr int kTmemCols = 512;
    static_assert(kAccCols + kAStages * kNA * 32 <= kTmemCols, "TMEM budget");
};

struct Barriers {
    uint64_t a_full[kMaxAStages];    // k-step dequantised into TMEM (one dequant group)
    uint64_t a_empty[kMaxAStages];   // MMAs reading that TMEM stage completed
    uint64_t b_full[8];           // token rows landed in shared memory (32 cp.async arrivals)
    uint64_t b_empty[8];
    uint64_t code_full[kMaxCodeChunks];
    uint64_t code_empty[kMaxCodeChunks];
    uint64_t meta_full[kMaxMetaBufs];
    uint64_t meta_empty[kMaxMetaBufs];
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
        if (e < p.E) {
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
    // exclusive scan of the per-thread tile counts: warp shuffles, then one
    // warp over the warp totals
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off)
            incl += v;
    }
    if (lane == 31)
        s_part[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kThreads / 32 ? s_part[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xFFFFFFFFu, w, off);
            if (lane >= off)
                w += v;
        }
        s_part[32 + lane] = w;   // inclusive prefix of the warp totals
    }
    __syncthreads();
    int run = incl - local + (warp > 0 ? s_part[32 + warp - 1] : 0);
    for (int e = e0; e < min(n, e0 + per); ++e) {
        s_tile_start[e] = run;
        run += (s_row_count[e] + BN - 1) / BN;
    }
    if (threadIdx.x == kThreads - 1)
        s_tile_start[n] = s_part[32 + kThreads / 32 - 1];
}

template <int MODE, int WFMT, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ GemmArgs p, const __grid_constant__ CUtensorMap tmap_b,
                        const __grid_constant__ CUtensorMap tmap_b2)
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
    // code ring: NCS chunks of CK k-steps; meta ring: NMETA per-tile blocks
    const int CK = 1 << p.ck_log2, NCS = 1 << p.ncs_log2, NMETA = 1 << p.nmeta_log2;
    const int chunk_bytes = CK * L::kCodeBlock;
    uint8_t *sMeta = sCode + NCS * chunk_bytes;
    const int meta_bytes = p.meta_bytes;
    const int meta_al = (meta_bytes + 127) & ~127;
    Barriers *bars = (Barriers *)(sMeta + NMETA * meta_al);
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
        for (int s = 0; s < L::kAStages; ++s) {
            mbar_init(&bars->a_full[s], L::kGroupWarps);
            mbar_init(&bars->a_empty[s], 1);
        }
        for (int s = 0; s < L::kBStages; ++s) {
            mbar_init(&bars->b_full[s], 1);   // one arrival with the stage's byte count
            mbar_init(&bars->b_empty[s], 1);
        }
        for (int s = 0; s < NCS; ++s) {
            mbar_init(&bars->code_full[s], 1);
            mbar_init(&bars->code_empty[s], kDeqWarps);   // every dequant warp reads every chunk
        }
        for (int s = 0; s < NMETA; ++s) {
            mbar_init(&bars->meta_full[s], 1);
            mbar_init(&bars->meta_empty[s], kDeqWarps);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->acc_full[s], 1);
            mbar_init(&bars->acc_empty[s], 4);
        }
        mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        bars->never_abort = 0;
        fence_mbar_init();
    }
    // everything below reads what the previous kernels in the stream wrote
    pdl_wait();
    pdl_allow_successor();
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
    WaitCtx wc{&bars->abort_flag, p.status, globaltimer_ns(), wait_limit_ns(p.status)};
    CYC_DECL

    if (warp == 0) {
        // ------------------------------------------------ B producer (TMA tiles of contiguous rows)
        // A tile of BN rows from the unit's first row: rows of the next
        // expert only feed MMA columns the epilogue discards, rows past the
        // end of the source arrive as zeros.  With a second source (gate/up
        // with a shared expert) the shared expert's units read x itself.
        if (elect_one()) {
            tma_prefetch_desc(&tmap_b);
            if (p.b_src2)
                tma_prefetch_desc(&tmap_b2);
        }
        __syncwarp();
        int step = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
            const Unit un = decode_unit<BN>(u, p, sched);
            const bool second = p.b_src2 && un.e >= p.E;
            const CUtensorMap *map = second ? &tmap_b2 : &tmap_b;
            const int y = second ? un.row0 - p.Tk : un.row0;
            CYC(2);
            for (int ks = 0; ks < KS; ++ks, ++step) {
                const int s = step % L::kBStages;
                if (step >= L::kBStages && !warp_wait(&bars->b_empty[s], ((step / L::kBStages) & 1) ^ 1, wc, 1)) {
                    ok = false;
                    break;
                }
                CYC(0);
                if (elect_one()) {
                    mbar_arrive_expect_tx(&bars->b_full[s], (uint32_t)(kBN * 128));
                    tma_load_2d(sB + s * kBN * 128, map, ks * kKStep, y, &bars->b_full[s]);
                }
                __syncwarp();
                CYC(1);
                if (lane == 0)
                    TRACE_OTHER(0, step);
            }
        }
        drain_ring(bars->b_full, step, L::kBStages, p.status, 12, &bars->never_abort);
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (converged warp, one elected lane)
        int step = 0, uidx = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++uidx) {
            const Unit un = decode_unit<BN>(u, p, sched);
            // fp16-operand mode: fp16 weights and tokens
            const uint32_t idesc = WFMT == MOE_WFMT_INT4_SYM_F16 ? idesc_f16_f32(128, un.nmma)
                                                                 : idesc_bf16_f32(128, un.nmma);
            const int ab = uidx % L::kAccBufs;
            const uint32_t acc = tmem + ab * L::kNAcc * kBN;
            CYC(4);
            if (uidx >= L::kAccBufs) {
                if (!mbar_wait(&bars->acc_empty[ab], ((uidx / L::kAccBufs) & 1) ^ 1, wc, 2))
                    break;
                tc_fence_after();
            }
            CYC(0);
            for (int ks = 0; ks < KS; ++ks, ++step) {
                const int sa = step % L::kAStages, sb = step % L::kBStages;
                // every lane polls the same barriers, so the outcome is warp-uniform
                if (!mbar_wait(&bars->a_full[sa], (step / L::kAStages) & 1, wc, 3)) {
                    ok = false;
                    break;
                }
                CYC(1);
                if (!mbar_wait(&bars->b_full[sb], (step / L::kBStages) & 1, wc, 4)) {
                    ok = false;
                    break;
                }
                CYC(2);
                if (lane == 0)
                    TRACE_OTHER(9, step);
                tc_fence_after();
                const uint64_t bdesc0 = sdesc_kmajor_sw128(smem_u32(sB + sb * kBN * 128));
                const uint32_t a_base = tmem + L::kAccCols + sa * L::kNA * 32;
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bdesc = bdesc0 + (uint64_t)(kk * 2);   // +32 bytes along K
#pragma unroll
                        for (int m = 0; m < L::kNA; ++m) {
                            mma_ts_f16(acc + m * kBN, a_base + m * 32 + kk * 8, bdesc, idesc, (ks | kk) != 0);
                        }
                    }
                    mma_commit(&bars->a_empty[sa]);
                    mma_commit(&bars->b_empty[sb]);
                }
                __syncwarp();
                CYC(3);
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
        WaitCtx wd{&bars->never_abort, p.status, globaltimer_ns(), kWaitLimitNs};   // drain even after an abort
        warp_wait(&bars->drain, 0, wd, 5);
    } else if (warp == 2) {
        // ------------------------------------------------ code / meta producer (converged warp)
        // A unit's code blocks are contiguous in the kernel layout, so one bulk
        // copy moves CK k-steps: the copy engine's throughput is set by the
        // number of copies more than by their size.  (Under the status block's
        // test knob this CTA issues none, and its dequant waits run out.)
        if (!test_knob_hits_this_cta(p.status)) {
            int cidx = 0, munit = 0, nmeta = 0;   // cidx: code chunks issued; nmeta: meta blocks issued
            bool ok = true;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++munit) {
                const Unit un = decode_unit<BN>(u, p, sched);
                const size_t tile_id = (size_t)un.e * p.F + un.f;
                const int mb = munit & (NMETA - 1);
                if (munit >= NMETA &&
                    !warp_wait(&bars->meta_empty[mb], ((munit >> p.nmeta_log2) & 1) ^ 1, wc, 6))
                    break;
                if (elect_one()) {
                    mbar_arrive_expect_tx(&bars->meta_full[mb], meta_bytes);
                    bulk_g2s(sMeta + mb * meta_al, p.wmeta + tile_id * meta_bytes, meta_bytes, &bars->meta_full[mb]);
                }
                __syncwarp();
                ++nmeta;
                for (int c0 = 0; c0 < KS; c0 += CK, ++cidx) {
                    const int s = cidx & (NCS - 1);
                    if (cidx >= NCS && !warp_wait(&bars->code_empty[s], ((cidx >> p.ncs_log2) & 1) ^ 1, wc, 7)) {
                        ok = false;
                        break;
                    }
                    const uint32_t bytes = (uint32_t)(min(CK, KS - c0) * L::kCodeBlock);
                    if (elect_one()) {
                        mbar_arrive_expect_tx(&bars->code_full[s], bytes);
                        bulk_g2s(sCode + s * chunk_bytes, p.wq + (tile_id * KS + c0) * L::kCodeBlock, bytes,
                                 &bars->code_full[s]);
                    }
                    __syncwarp();
                    if (lane == 0)
                        TRACE_OTHER(1, cidx);
                }
            }
            drain_ring(bars->code_full, cidx, NCS, p.status, 13, &bars->never_abort);
            drain_ring(bars->meta_full, nmeta, NMETA, p.status, 14, &bars->never_abort);
        }
    } else if (warp == 3) {
#ifdef MOEQ4_TRACE
        // instrumented builds, first CTAs: record when each code chunk lands
        // (event 14, by chunk), each B stage lands (event 8, by step) and each
        // A stage is complete in TMEM (event 10, by step)
        if (blockIdx.x < 4 && lane == 0) {
            int n_units = 0;
            for (int u = blockIdx.x; u < total_units; u += gridDim.x)
                ++n_units;
            const int n_chunks = n_units * ((KS + CK - 1) / CK), n_steps = n_units * KS;
            int ci = 0, bi = 0, ai = 0;
            uint64_t t_last = globaltimer_ns();
            auto test = [](uint32_t bar, uint32_t par) {
                uint32_t done;
                asm volatile("{\n\t.reg .pred q;\n\t"
                             "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 q, [%1], %2;\n\t"
                             "selp.u32 %0, 1, 0, q;\n\t}"
                             : "=r"(done) : "r"(bar), "r"(par) : "memory");
                return done != 0;
            };
            while ((ci < n_chunks || bi < n_steps || ai < n_steps) && globaltimer_ns() - t_last < 200000) {
                if (ci < n_chunks && test(smem_u32(&bars->code_full[ci & (NCS - 1)]), (ci >> p.ncs_log2) & 1)) {
                    TRACE_EVENT(14, ci);
                    ++ci;
                    t_last = globaltimer_ns();
                }
                if (bi < n_steps && test(smem_u32(&bars->b_full[bi % L::kBStages]), (bi / L::kBStages) & 1)) {
                    TRACE_EVENT(8, bi);
                    ++bi;
                    t_last = globaltimer_ns();
                }
                if (ai < n_steps && test(smem_u32(&bars->a_full[ai % L::kAStages]), (ai / L::kAStages) & 1)) {
                    TRACE_EVENT(10, ai);
                    ++ai;
                    t_last = globaltimer_ns();
                }
            }
        }
#endif
    } else if (warp >= 4 && warp < 4 + kDeqWarps) {
        // ------------------------------------------------ dequant into TMEM
        // Groups of L::kGroupWarps warps take k-steps round-robin; a warp owns
        // TMEM lane quadrant warp % 4 (32 weight rows) and L::kHalves of the
        // two 32-element halves of each of its k-steps.
        const int dw = warp - 4;
        const int grp = dw / L::kGroupWarps;              // k-steps with step % kGroups == grp
        const int c0 = L::kHalves == 1 ? (dw & 7) >> 2 : 0;
        const int r = (warp & 3) * 32 + lane;             // tile row == TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const int gshift = __ffs(max(p.G, 1)) - 1;        // int4-sym groups are a power of two
        int step = 0, munit = 0, cbase = 0;               // cbase: code chunk index of the unit's first k-step
        bool ok = true;
        for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++munit) {
            const int mb = munit & (NMETA - 1);
            const uint8_t *meta = sMeta + mb * meta_al;
            if (!mbar_wait(&bars->meta_full[mb], (munit >> p.nmeta_log2) & 1, wc, 8))
                break;
            CYC(7);
            const int ngroups = WFMT == MOE_WFMT_Q4K ? p.K / 256 : p.K >> gshift;
            // This warp's k-steps of the unit: those with step % kGroups == grp.
            // Every dequant warp frees every code chunk of the unit exactly
            // once: right after its last k-step in the chunk, or, for chunks
            // where it has none, as it passes them.
            const int step0 = step;                       // global step of k-step 0
            const int nchunks = (KS + CK - 1) >> p.ck_log2;
            int released = 0;                             // chunks of this unit already freed
            for (int ks = ((grp - step0) % L::kGroups + L::kGroups) % L::kGroups; ks < KS; ks += L::kGroups) {
                step = step0 + ks;
                const int sa = step % L::kAStages;
                const uint32_t a_col = tmem + lane_off + L::kAccCols + sa * L::kNA * 32;
                CYC(6);
                const int my_chunk = ks >> p.ck_log2;
                const int cidx = cbase + my_chunk;
                const int sc = cidx & (NCS - 1);
                // chunks passed without a k-step of this warp are freed before it
                // waits for a later one (a warp never holds one chunk while
                // waiting for another)
                if (my_chunk > released) {
                    __syncwarp();
                    if (lane == 0)
                        for (int cc = released; cc < my_chunk; ++cc)
                            mbar_arrive(&bars->code_empty[(cbase + cc) & (NCS - 1)]);
                    released = my_chunk;
                }
                if (lane == 0 && warp == 4)
                    TRACE_OTHER(15, step);
                if (!mbar_wait(&bars->code_full[sc], (cidx >> p.ncs_log2) & 1, wc, 9)) {
                    ok = false;
                    break;
                }
                CYC(0);
#ifdef MOEQ4_TRACE_WARPS
                if (lane == 0)
                    TRACE_EVENT((warp - 4) * 2, step);
#else
                if (lane == 0 && warp == 4)
                    TRACE_EVENT(2, step);
#endif
                const uint32_t cblk = smem_u32(sCode) + sc * chunk_bytes + (ks & (CK - 1)) * L::kCodeBlock;
#pragma unroll 1
                for (int h = 0; h < L::kHalves; ++h) {
                    const int c = c0 + h;
                    const int kpos = ks * kKStep + c * 32;
                    uint32_t words[L::kNA][16];
#pragma unroll
                    for (int m = 0; m < L::kNA; ++m) {
                        const uint4 codes = lds128(cblk + ((m * 2 + c) * kTileRows + r) * kChunkBytes);
                        if (WFMT == MOE_WFMT_Q4K) {
                            const int g = kpos / 256;
                            const uint4 hdr = lds128(smem_u32(meta) + ((m * ngroups + g) * kTileRows + r) * 16);
                            float dsc, dm;
                            q4k_subblock_scale(hdr, (kpos % 256) / 32, dsc, dm);
                            dequant_q4k_chunk(codes, dsc, dm, words[m]);
                        } else if (WFMT == MOE_WFMT_INT4_ASYM) {
                            const int g = kpos >> gshift;
                            const uint32_t sm = lds32(smem_u32(meta) + ((m * ngroups + g) * kTileRows + r) * 4);
                            dequant_int4asym_chunk(codes, sm, words[m]);
                        } else if (WFMT == MOE_WFMT_INT4_SYM_F16) {
                            const int g = kpos >> gshift;
                            const uint16_t sbits = lds16(smem_u32(meta) + ((m * ngroups + g) * kTileRows + r) * 2);
                            dequant_int4sym_f16_chunk(codes, sbits, words[m]);
                        } else {
                            const int g = kpos >> gshift;
                            const uint16_t sbits = lds16(smem_u32(meta) + ((m * ngroups + g) * kTileRows + r) * 2);
                            dequant_int4sym_chunk(codes, sbits, words[m]);
                        }
                    }
                    if (h == 0) {
                        CYC(1);
                        if (lane == 0 && warp == 4)
                            TRACE_EVENT(11, step);
                        // the MMAs that read this TMEM stage kAStages k-steps ago have finished
                        if (step >= L::kAStages &&
                            !mbar_wait(&bars->a_empty[sa], ((step / L::kAStages) & 1) ^ 1, wc, 10)) {
                            ok = false;
                            break;
                        }
                        if (lane == 0 && warp == 4)
                            TRACE_OTHER(12, step);
                        tc_fence_after();
                        CYC(2);
                    }
#pragma unroll
                    for (int m = 0; m < L::kNA; ++m)
                        tmem_st16(a_col + m * 32 + c * 16, words[m]);
                    CYC(h == 0 ? 3 : 4);
                }
                if (!ok)
                    break;
                // after its last k-step in the chunk the warp frees it
                const int chunk_end = min((my_chunk + 1) << p.ck_log2, KS);
                if (ks + L::kGroups >= chunk_end) {
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&bars->code_empty[sc]);
                    released = my_chunk + 1;
                }
                CYC(11);
                tmem_wait_st();
                CYC(5);
                if (lane == 0 && warp == 4)
                    TRACE_OTHER(13, step);
                tc_fence_before();
                __syncwarp();
                CYC(9);
                if (lane == 0)
                    mbar_arrive(&bars->a_full[sa]);
                __syncwarp();
                CYC(10);
                if (lane == 0 && warp == 4)
                    TRACE_OTHER(3, step);
                if (lane == 0 && warp == 7)
                    TRACE_OTHER(4, step);
            }
            if (!ok)
                break;
            step = step0 + KS;
            __syncwarp();
            if (lane == 0) {
                for (int cc = released; cc < nchunks; ++cc)
                    mbar_arrive(&bars->code_empty[(cbase + cc) & (NCS - 1)]);
                mbar_arrive(&bars->meta_empty[mb]);
            }
            cbase += (KS + CK - 1) >> p.ck_log2;
        }
    } else {
        // ------------------------------------------------ epilogue (last four warps)
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        int uidx = 0;
        for (int u = blockIdx.x; u < total_units; u += gridDim.x, ++uidx) {
            const Unit un = decode_unit<BN>(u, p, sched);
            const int ab = uidx % L::kAccBufs;
            CYC(1);
            if (!mbar_wait(&bars->acc_full[ab], (uidx / L::kAccBufs) & 1, wc, 11))
                break;
            CYC(0);
            tc_fence_after();
            if (lane == 0 && warp == 4 + kDeqWarps)
                TRACE_OTHER(6, uidx);
            const uint32_t acc = tmem + lane_off + ab * L::kNAcc * kBN;
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
                    // h is fp16 in the fp16-operand mode (the down pass's operand); Y is bf16
                    if (MODE == MODE_GATE_UP && WFMT == MOE_WFMT_INT4_SYM_F16)
                        *(__half *)(stage + j * kEpiStride + lane * 2) = __float2half_rn(o);
                    else
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
            if (!released) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars->acc_empty[ab]);
            }
            if (lane == 0 && warp == 4 + kDeqWarps)
                TRACE_OTHER(7, uidx);
        }
    }

    CYC(7);
    CYC_FLUSH;
#ifdef MOEQ4_TRACE
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (wc.waits[i]) {
                atomicAdd(&g_wait_stats[i][0], (unsigned long long)wc.waits[i]);
                atomicAdd(&g_wait_stats[i][1], (unsigned long long)wc.polls[i]);
            }
        }
    }
#endif
    __syncthreads();
    if (warp == 3) {
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
    }
}

constexpr size_t kSmemLimit = 227 * 1024;

// Shared-memory ring configuration of one launch (all counts are powers of two).
struct Rings {
    int ck_log2, ncs_log2, nmeta_log2;
};

template <int MODE, int BN>
static size_t gemm_smem_bytes(int meta_bytes, int E_total, const Rings &r)
{
    using L = Geo<MODE, BN>;
    const size_t code = ((size_t)L::kCodeBlock << r.ck_log2) << r.ncs_log2;
    const size_t need = 1024 + L::kBBytes + code + ((size_t)((meta_bytes + 127) & ~127) << r.nmeta_log2) +
                        sizeof(Barriers) + sizeof(int) * (3 * E_total + 1 + kThreads) + 16 + kEpiBytes;
    // at least half of the SM's shared memory, so that one CTA (and one TMEM
    // allocation) runs per SM
    return need > 116 * 1024 ? need : 116 * 1024;
}

// Code chunks of up to 32 KB (CK k-steps per bulk copy) and as many chunks in
// flight (up to 8, at least 4 where possible) as shared memory holds; four
// meta blocks in flight when they are small.
template <int MODE, int BN>
static Rings gemm_rings(int meta_bytes, int E_total, int KS)
{
    using L = Geo<MODE, BN>;
    Rings r{0, 0, 1};
    r.nmeta_log2 = meta_bytes <= 4096 ? 2 : 1;
    r.ck_log2 = 1;
    while ((L::kCodeBlock << (r.ck_log2 + 1)) <= 32768 && (1 << (r.ck_log2 + 1)) <= KS)
        ++r.ck_log2;
    for (;;) {
        r.ncs_log2 = 3;
        while (r.ncs_log2 > 1 && gemm_smem_bytes<MODE, BN>(meta_bytes, E_total, r) > kSmemLimit)
            --r.ncs_log2;
        if (r.ncs_log2 >= 2 || r.ck_log2 == 1)
            break;
        --r.ck_log2;
    }
    return r;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda); null if the driver does not provide it.
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
        return (PFN_cuTensorMapEncodeTiled_v12000)f;
    }();
    return fn;
}

// Tensor map of the B rows (bf16 [b_rows, ldb], row-major) in tiles of
// 64 elements (128 bytes, 128-byte swizzle: the MMA's K-major layout) by
// BN rows.
cudaError_t encode_b_map(CUtensorMap *m, const uint16_t *src, int ld, int rows, int bn)
{
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc)
        return cudaErrorNotSupported;
    if ((reinterpret_cast<uintptr_t>(src) & 15) || rows < 1 || ((size_t)ld * 2) % 16)
        return cudaErrorInvalidValue;
    const cuuint64_t dims[2] = {(cuuint64_t)ld, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kKStep, (cuuint32_t)bn};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(src), dims, strides,
                           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_kstep_map(CUtensorMap *m, const uint16_t *src, int ld, int rows, int box_rows, int box_ksteps)
{
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc)
        return cudaErrorNotSupported;
    if ((reinterpret_cast<uintptr_t>(src) & 15) || rows < 1 || ld % kKStep || box_ksteps < 1 ||
        box_ksteps > ld / kKStep || box_rows < 8 || box_rows > 256)
        return cudaErrorInvalidValue;
    const cuuint64_t dims[3] = {(cuuint64_t)kKStep, (cuuint64_t)rows, (cuuint64_t)(ld / kKStep)};
    const cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)kKStep * 2};
    const cuuint32_t box[3] = {(cuuint32_t)kKStep, (cuuint32_t)box_rows, (cuuint32_t)box_ksteps};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t *>(src), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int MODE, int WFMT, int BN>
static cudaError_t launch_one(const GemmArgs &a_in, int num_sms, cudaStream_t st)
{
    auto kern = grouped_gemm_kernel<MODE, WFMT, BN>;
    CUtensorMap tmap{}, tmap2{};
    cudaError_t e = encode_b_map(&tmap, a_in.b_src, a_in.ldb, a_in.b_rows, BN);
    if (e == cudaSuccess && a_in.b_src2)
        e = encode_b_map(&tmap2, a_in.b_src2, a_in.ldb, a_in.b_rows2, BN);
    if (e != cudaSuccess)
        return e;
    GemmArgs a = a_in;
    const Rings r = gemm_rings<MODE, BN>(a.meta_bytes, a.E_total, a.K / kKStep);
    a.ck_log2 = r.ck_log2;
    a.ncs_log2 = r.ncs_log2;
    a.nmeta_log2 = r.nmeta_log2;
    const size_t smem = gemm_smem_bytes<MODE, BN>(a.meta_bytes, a.E_total, r);
    if (smem > kSmemLimit)
        return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    return launch_pdl(kern, num_sms, kThreads, smem, st, a, tmap, tmap2);
}

size_t gemm_smem_required(int nmat, int meta_bytes, int E_total)
{
    // the smallest rings (two chunks of two k-steps, two meta blocks) of the larger tile
    const Rings r{1, 1, 1};
    const size_t a = nmat == 2 ? gemm_smem_bytes<MODE_GATE_UP, 64>(meta_bytes, E_total, r)
                               : gemm_smem_bytes<MODE_DOWN, 64>(meta_bytes, E_total, r);
    const size_t b = nmat == 2 ? gemm_smem_bytes<MODE_GATE_UP, 192>(meta_bytes, E_total, r)
                               : gemm_smem_bytes<MODE_DOWN, 256>(meta_bytes, E_total, r);
    const size_t c = nmat == 2 ? gemm_smem_bytes<MODE_GATE_UP, 128>(meta_bytes, E_total, r) : 0;
    return a > b ? (a > c ? a : c) : (b > c ? b : c);
}

// Gate/up token tiles: 64 when experts average at most 64 rows; when they
// average at least 128, 192 (one accumulator of 2 x 192 columns and two A
// stages fill TMEM: half again the MMA work per dequantised k-step), or 160
// for Q4K super-blocks, whose heavier dequantisation gains more from a
// third A stage than from the wider tile (measured: 4096 tokens 266 -> 257
// us; int4-sym at 8192 tokens prefers 192, 397 vs 425 us); else 128.
#ifndef MOEQ4_GU_TILE_MAX
#define MOEQ4_GU_TILE_MAX 192
#endif
int gemm_tile_tokens(int T, int E, int k, int wfmt)
{
    if ((long long)T * k <= 64LL * E)
        return 64;
    if (MOEQ4_GU_TILE_MAX < 192 || (long long)T * k < 128LL * E)
        return 128;
    return wfmt == MOE_WFMT_Q4K ? 160 : 192;
}

// The down pass reads its token rows with TMA and has a single matrix, so
// when experts average at least 128 rows it takes 256-token tiles: twice the
// MMA work per dequantised k-step and per pipeline round trip.
#ifndef MOEQ4_DOWN_TILE_MAX
#define MOEQ4_DOWN_TILE_MAX 256
#endif
int gemm_down_tile_tokens(int T, int E, int k)
{
    if (MOEQ4_DOWN_TILE_MAX >= 256 && (long long)T * k >= 128LL * E)
        return 256;
    return (long long)T * k <= 64LL * E ? 64 : 128;
}

template <int MODE, int BN>
static cudaError_t launch_fmt(const GemmArgs &a, int wfmt, int num_sms, cudaStream_t st)
{
    return wfmt == MOE_WFMT_Q4K             ? launch_one<MODE, MOE_WFMT_Q4K, BN>(a, num_sms, st)
           : wfmt == MOE_WFMT_INT4_ASYM     ? launch_one<MODE, MOE_WFMT_INT4_ASYM, BN>(a, num_sms, st)
           : wfmt == MOE_WFMT_INT4_SYM_F16 ? launch_one<MODE, MOE_WFMT_INT4_SYM_F16, BN>(a, num_sms, st)
                                            : launch_one<MODE, MOE_WFMT_INT4_SYM, BN>(a, num_sms, st);
}

cudaError_t launch_grouped_gemm(const GemmArgs &a, int nmat, int wfmt, int tile_tokens, int num_sms, cudaStream_t st)
{
    if (nmat == 2)
        return tile_tokens == 64    ? launch_fmt<MODE_GATE_UP, 64>(a, wfmt, num_sms, st)
               : tile_tokens == 192 ? launch_fmt<MODE_GATE_UP, 192>(a, wfmt, num_sms, st)
               : tile_tokens == 160 ? launch_one<MODE_GATE_UP, MOE_WFMT_Q4K, 160>(a, num_sms, st)
                                    : launch_fmt<MODE_GATE_UP, 128>(a, wfmt, num_sms, st);
    return tile_tokens == 64    ? launch_fmt<MODE_DOWN, 64>(a, wfmt, num_sms, st)
           : tile_tokens == 128 ? launch_fmt<MODE_DOWN, 128>(a, wfmt, num_sms, st)
                                : launch_fmt<MODE_DOWN, 256>(a, wfmt, num_sms, st);
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
    static unsigned long long zero_w[16 * 2];
    cudaError_t e = cudaMemcpyToSymbol(g_wait_stats, zero_w, sizeof(zero_w));
    if (e == cudaSuccess)
        e = cudaMemcpyToSymbol(moeq4::g_trace, zero, sizeof(zero));
    return (int)e;
}
extern "C" int moe_cyc_fetch(unsigned long long *host)
{
    return (int)cudaMemcpyFromSymbol(host, g_cyc, sizeof(g_cyc));
}
extern "C" int moe_wait_stats_fetch(unsigned long long *host)
{
    return (int)cudaMemcpyFromSymbol(host, g_wait_stats, sizeof(g_wait_stats));
}
#endif
