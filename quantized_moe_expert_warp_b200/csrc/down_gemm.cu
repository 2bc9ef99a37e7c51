// Grouped down GEMM with the dequantised weight tile resident in TMEM.
//
// The down projection of an expert is Y[token, :] = h[token, :] Wd^T with
// Wd [H, I] in 4-bit codes (hipfire 0.4.3 benchmarks, "Read this before
// comparing columns": the MoE prefill route; the B200 counterpart of its
// per-expert GEMMs).  With K = I <= 512, one 128-row tile of Wd, expanded to
// bf16 (or fp16), fills at most 256 TMEM columns: it is dequantised once and
// then multiplied with every token tile of a work item (up to `item_tiles`
// tiles of BN tokens of the same expert), instead of once per token tile.
// The remaining 256 columns hold two BN-column accumulators, so the
// epilogue of one token tile runs under the MMAs of the next.
//
// TMEM A slots are k-steps (64 elements of K, 32 columns): the MMAs of an
// item's last token tile release them one by one, and the dequant warps
// refill each slot for the next item as soon as it is free, so the next
// item's weights are expanded while the current one's last MMAs run.
//
// Work items (expert, 128-row tile f, up to item_tiles token tiles) are
// taken in a fixed order that every CTA derives from the permutation
// offsets: items of item_tiles full tiles first, then the experts' last
// items by decreasing tile count (longest first), each item's F row tiles
// consecutively.  CTA b takes units b, b + grid, ...
//
// Warp roles (768 threads, one CTA per SM):
//   warp 0      B producer (one lane): per ring stage one TMA copy of
//               `b_sk` k-steps of h rows (32, 64 or 128 rows, the smallest
//               box that covers the tile's MMA width)
//   warp 1      MMA issuer (one elected thread)
//   warp 2      code and scale blocks of each item, one bulk copy each
//   warp 3      TMEM allocation
//   warps 4-15  dequant: three groups of four warps; group g expands k-steps
//               g, g + 3, ...; warp % 4 is the TMEM lane quadrant (32 rows)
//   warps 16-23 epilogue (TMEM -> bf16 -> y rows): two warps per lane
//               quadrant take alternate 16-column chunks of a token tile, so
//               that draining a tile takes no longer than its MMAs
// Every wait is bounded; on timeout the CTA records MOE_ERR_TIMEOUT and
// unwinds.
//
// A ring stage carries several k-steps (up to 64 KB) on one barrier: on
// this hardware a copy engine completes about one barrier phase per 300 ns
// per SM however small the copy, so 16 KB stages cap the feed near 50 GB/s
// per SM while 64 KB stages reach about 130 GB/s.  The copies are issued
// by a single lane; issuing and waiting from a converged warp with an
// elected lane measured about twice as slow per stage.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "dequant.cuh"
#include "kernels.h"
#include "moeq4.h"
#include "ptx.cuh"

namespace moeq4 {

namespace {

constexpr int kDnThreads = 768;
constexpr int kDnDeqWarps = 12;
constexpr int kDnGroups = 3;
constexpr int kDnEpiWarps = 8;
static_assert(4 + kDnDeqWarps + kDnEpiWarps == kDnThreads / 32, "warp roles");
constexpr int kDnMaxKS = 8;          // A slots: K <= 512
constexpr int kDnMaxBStages = 4;
constexpr int kDnMaxNCS = 2;         // code blocks of items in flight
constexpr int kDnMaxMeta = 4;
constexpr int kDnEpiTok = 16;
constexpr int kDnEpiStride = 80;
constexpr int kDnEpiBytes = kDnEpiWarps * kDnEpiTok * kDnEpiStride;
constexpr int kDnCodeStep = code_block_bytes(1);   // 4 KB: one k-step of a 128-row tile

struct DnBars {
    uint64_t a_full[kDnMaxKS];
    uint64_t a_empty[kDnMaxKS];
    uint64_t b_full[kDnMaxBStages];
    uint64_t b_empty[kDnMaxBStages];
    uint64_t code_full[kDnMaxNCS];
    uint64_t code_empty[kDnMaxNCS];
    uint64_t meta_full[kDnMaxMeta];
    uint64_t meta_empty[kDnMaxMeta];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int never_abort;
    int n_full;   // items of item_tiles full tiles
    int n_rem;    // remainder items
};

// The schedule in shared memory.
struct DnSched {
    int *row_start;    // [E_total] first permuted row of each expert
    int *row_count;    // [E_total]
    int *full_start;   // [E_total + 1] prefix of the experts' full-item counts
    int *rem_e;        // [E_total] experts of the remainder items, in order
};

struct DnItem {
    int e, f, row0, rows, ntiles;
};

template <int BN>
__device__ __forceinline__ DnItem dn_item(int u, const GemmArgs &p, const DnSched &s, int n_full)
{
    DnItem it;
    const int i = u / p.F;
    it.f = u - i * p.F;
    const int NT = p.item_tiles;
    int tile0;
    if (i < n_full) {
        int lo = 0, hi = p.E_total - 1;   // largest e with full_start[e] <= i
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s.full_start[mid] <= i)
                lo = mid;
            else
                hi = mid - 1;
        }
        it.e = lo;
        tile0 = (i - s.full_start[lo]) * NT;
    } else {
        it.e = s.rem_e[i - n_full];
        tile0 = (s.full_start[it.e + 1] - s.full_start[it.e]) * NT;
    }
    const int n = s.row_count[it.e];
    it.row0 = s.row_start[it.e] + tile0 * BN;
    it.rows = min(NT * BN, n - tile0 * BN);
    it.ntiles = (it.rows + BN - 1) / BN;
    return it;
}

__device__ __forceinline__ int mma_width(int nvalid) { return max(16, (nvalid + 15) & ~15); }

// TMA box (index into the kernel's maps: 32, 64, 128 rows) for an MMA width
__device__ __forceinline__ int box_index(int nmma) { return nmma <= 32 ? 0 : nmma <= 64 ? 1 : 2; }

// Builds the schedule.  Rows of expert e are [offsets[e], offsets[e+1]);
// the shared expert (if any) is expert E with rows [T k, T k + T).  Expert
// e has t = ceil(rows / BN) token tiles: t / NT full items and, when t % NT
// > 0, one remainder item.  Warp 0 writes the full-item prefix; warp w =
// 1 .. NT - 1 lists the experts whose remainder has NT - w tiles, in expert
// order, after those of longer remainders.
template <int BN>
__device__ void dn_build_schedule(const GemmArgs &p, const DnSched &s, DnBars *bars, int *s_bucket)
{
    const int n = p.E_total, NT = p.item_tiles;
    for (int e = threadIdx.x; e < n; e += kDnThreads) {
        int start, cnt;
        if (e < p.E) {
            start = p.offsets[e];
            cnt = p.offsets[e + 1] - p.offsets[e];
        } else {
            start = p.Tk;
            cnt = p.T;
        }
        s.row_start[e] = start;
        s.row_count[e] = cnt;
    }
    if (threadIdx.x < 32)
        s_bucket[threadIdx.x] = 0;
    __syncthreads();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // remainder sizes per bucket (atomics only count; the order comes from ballots below)
    for (int e = threadIdx.x; e < n; e += kDnThreads) {
        const int r = ((s.row_count[e] + BN - 1) / BN) % NT;
        if (r)
            atomicAdd(&s_bucket[r], 1);
    }
    __syncthreads();
    if (warp == 0) {
        int run = 0;
        for (int c = 0; c < n; c += 32) {
            const int e = c + lane;
            const int q = e < n ? ((s.row_count[e] + BN - 1) / BN) / NT : 0;
            int incl = q;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (lane >= off)
                    incl += v;
            }
            if (e < n)
                s.full_start[e] = run + incl - q;
            run += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0) {
            s.full_start[n] = run;
            bars->n_full = run;
            int tot = 0;
            for (int r = 1; r < NT; ++r)
                tot += s_bucket[r];
            bars->n_rem = tot;
        }
    } else if (warp < NT) {
        const int r = NT - warp;   // this warp's remainder size
        int pos = 0;               // items of longer remainders come first
        for (int rr = NT - 1; rr > r; --rr)
            pos += s_bucket[rr];
        for (int c = 0; c < n; c += 32) {
            const int e = c + lane;
            const bool mine = e < n && ((s.row_count[e] + BN - 1) / BN) % NT == r;
            const unsigned m = __ballot_sync(0xFFFFFFFFu, mine);
            if (mine)
                s.rem_e[pos + __popc(m & ((1u << lane) - 1u))] = e;
            pos += __popc(m);
        }
    }
    __syncthreads();
}

template <int WFMT, int BN, int SK>
__global__ void __launch_bounds__(kDnThreads, 1)
    down_resident_kernel(const __grid_constant__ GemmArgs p, const __grid_constant__ CUtensorMap tmap32,
                         const __grid_constant__ CUtensorMap tmap64, const __grid_constant__ CUtensorMap tmap128)
{
    constexpr int kAccCols = 2 * BN;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int KS = p.K / kKStep;
    const int NB = p.b_stages;                // B ring depth
    const int stage_bytes = BN * 128 * SK;
    const int NCS = p.ncs;                    // code ring depth (items)
    const int NMETA = p.nmeta;
    const int item_code = KS * kDnCodeStep;   // code bytes of one item
    const int meta_bytes = p.meta_bytes;
    const int meta_al = (meta_bytes + 127) & ~127;
    uint8_t *sB = smem;
    uint8_t *sCode = sB + NB * stage_bytes;
    uint8_t *sMeta = sCode + NCS * item_code;
    DnBars *bars = (DnBars *)(sMeta + NMETA * meta_al);
    int *s_bucket = (int *)(bars + 1);
    DnSched sched;
    sched.row_start = s_bucket + 32;
    sched.row_count = sched.row_start + p.E_total;
    sched.full_start = sched.row_count + p.E_total;
    sched.rem_e = sched.full_start + p.E_total + 1;
    uint8_t *s_epi = (uint8_t *)(sched.rem_e + p.E_total);
    s_epi += (16u - (smem_u32(s_epi) & 15u)) & 15u;

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < KS; ++s) {
            mbar_init(&bars->a_full[s], 4);   // the four warps of a dequant group
            mbar_init(&bars->a_empty[s], 1);
        }
        for (int s = 0; s < NB; ++s) {
            mbar_init(&bars->b_full[s], 1);
            mbar_init(&bars->b_empty[s], 1);
        }
        for (int s = 0; s < NCS; ++s) {
            mbar_init(&bars->code_full[s], 1);
            mbar_init(&bars->code_empty[s], kDnDeqWarps);
        }
        for (int s = 0; s < NMETA; ++s) {
            mbar_init(&bars->meta_full[s], 1);
            mbar_init(&bars->meta_empty[s], kDnDeqWarps);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->acc_full[s], 1);
            mbar_init(&bars->acc_empty[s], kDnEpiWarps);
        }
        mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        bars->never_abort = 0;
        fence_mbar_init();
    }
    pdl_wait();
    pdl_allow_successor();
    dn_build_schedule<BN>(p, sched, bars, s_bucket);
    if (warp == 3) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const int n_full = bars->n_full;
    const int total = (n_full + bars->n_rem) * p.F;
    WaitCtx wc{&bars->abort_flag, p.status, globaltimer_ns(), wait_limit_ns(p.status)};

    if (warp == 0) {
        // ------------------------------------------------ B producer (lane 0 alone)
        if (lane == 0) {
            tma_prefetch_desc(&tmap32);
            tma_prefetch_desc(&tmap64);
            tma_prefetch_desc(&tmap128);
            int stage = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
                const DnItem it = dn_item<BN>(u, p, sched, n_full);
                for (int j = 0; j < it.ntiles && ok; ++j) {
                    const int nmma = mma_width(min(BN, it.rows - j * BN));
                    const int bx = box_index(nmma);
                    const CUtensorMap *map = bx == 0 ? &tmap32 : bx == 1 ? &tmap64 : &tmap128;
                    const uint32_t bytes = (uint32_t)(32 << bx) * 128u * (uint32_t)SK;
                    for (int k0 = 0; k0 < KS; k0 += SK, ++stage) {
                        const int s = stage % NB;
                        if (stage >= NB && !mbar_wait(&bars->b_empty[s], ((stage / NB) & 1) ^ 1, wc, 41)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&bars->b_full[s], bytes);
                        tma_load_3d(sB + s * stage_bytes, map, 0, it.row0 + j * BN, k0, &bars->b_full[s]);
                    }
                }
            }
            drain_ring_lane(bars->b_full, stage, NB, p.status, 42, &bars->never_abort);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        int tidx = 0, iidx = 0;
        int sb = 0;            // B ring slot of the next stage
        uint32_t bpar = 0;     // and the parity of its phase
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x, ++iidx) {
            const DnItem it = dn_item<BN>(u, p, sched, n_full);
            for (int j = 0; j < it.ntiles && ok; ++j, ++tidx) {
                const int nmma = mma_width(min(BN, it.rows - j * BN));
                const uint32_t idesc = WFMT == MOE_WFMT_INT4_SYM_F16 ? idesc_f16_f32(128, nmma) : idesc_bf16_f32(128, nmma);
                const int ab = tidx & 1;
                const uint32_t acc = tmem + ab * BN;
                if (tidx >= 2) {
                    if (!mbar_wait(&bars->acc_empty[ab], ((tidx >> 1) & 1) ^ 1, wc, 43)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                const bool last = j == it.ntiles - 1;
                const int box_rows = 32 << box_index(nmma);   // rows per k-step slab of the stage
                for (int k0 = 0; k0 < KS && ok; k0 += SK) {
                    if (!mbar_wait(&bars->b_full[sb], bpar, wc, 45)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sbase = smem_u32(sB + sb * stage_bytes);
                    if (j == 0) {
                        // first tile of the item: the stage's weight slots must be filled
#pragma unroll
                        for (int t = 0; t < SK; ++t)
                            if (ok && !mbar_wait(&bars->a_full[k0 + t], iidx & 1, wc, 44))
                                ok = false;
                        if (!ok)
                            break;
                    }
                    // the stage's SK x 4 MMAs straight from one elected lane (issue cost,
                    // not the tensor pipe, bounds a loop with per-k-step bookkeeping at N = 128)
                    tc_fence_after();
                    if (elect_one()) {
                        const uint64_t d0 = sdesc_kmajor_sw128(sbase);
                        const uint32_t a0 = tmem + kAccCols + k0 * 32;
                        const uint32_t slab = (uint32_t)(box_rows * 8);   // descriptor units of a k-step slab
#pragma unroll
                        for (int t = 0; t < SK; ++t)
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_ts_f16(acc, a0 + t * 32 + kk * 8, d0 + (uint64_t)(t * slab + kk * 2), idesc,
                                           (t | kk) ? 1u : (uint32_t)k0);
                        if (last) {   // the item's weights in these slots are no longer needed
#pragma unroll
                            for (int t = 0; t < SK; ++t)
                                mma_commit(&bars->a_empty[k0 + t]);
                        }
                        mma_commit(&bars->b_empty[sb]);
                    }
                    __syncwarp();
                    if (++sb == NB) {
                        sb = 0;
                        bpar ^= 1u;
                    }
                }
                if (ok) {
                    if (elect_one())
                        mma_commit(&bars->acc_full[ab]);
                    __syncwarp();
                }
            }
        }
        if (elect_one())
            mma_commit(&bars->drain);
        __syncwarp();
        WaitCtx wd{&bars->never_abort, p.status, globaltimer_ns(), kWaitLimitNs};
        warp_wait(&bars->drain, 0, wd, 46);
    } else if (warp == 2) {
        // ------------------------------------------------ code / scale producer (under the
        // status block's test knob this CTA issues none, and its dequant waits run out)
        if (!test_knob_hits_this_cta(p.status)) {
            int iidx = 0, nmeta = 0, ncode = 0;   // items seen, scale and code blocks issued
            for (int u = blockIdx.x; u < total; u += gridDim.x, ++iidx) {
                const DnItem it = dn_item<BN>(u, p, sched, n_full);
                const size_t tile_id = (size_t)it.e * p.F + it.f;
                const int mb = iidx % NMETA, cs = iidx % NCS;
                if (iidx >= NMETA && !warp_wait(&bars->meta_empty[mb], ((iidx / NMETA) & 1) ^ 1, wc, 47))
                    break;
                if (elect_one()) {
                    mbar_arrive_expect_tx(&bars->meta_full[mb], (uint32_t)meta_bytes);
                    bulk_g2s(sMeta + mb * meta_al, p.wmeta + tile_id * meta_bytes, (uint32_t)meta_bytes,
                             &bars->meta_full[mb]);
                }
                __syncwarp();
                ++nmeta;
                if (iidx >= NCS && !warp_wait(&bars->code_empty[cs], ((iidx / NCS) & 1) ^ 1, wc, 48))
                    break;
                if (elect_one()) {
                    mbar_arrive_expect_tx(&bars->code_full[cs], (uint32_t)item_code);
                    bulk_g2s(sCode + cs * item_code, p.wq + tile_id * item_code, (uint32_t)item_code,
                             &bars->code_full[cs]);
                }
                __syncwarp();
                ++ncode;
            }
            drain_ring(bars->meta_full, nmeta, NMETA, p.status, 49, &bars->never_abort);
            drain_ring(bars->code_full, ncode, NCS, p.status, 50, &bars->never_abort);
        }
    } else if (warp >= 4 && warp < 4 + kDnDeqWarps) {
        // ------------------------------------------------ dequant into the TMEM A slots
        const int grp = (warp - 4) / 4;
        const int r = (warp & 3) * 32 + lane;   // tile row == TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const int gshift = __ffs(max(p.G, 1)) - 1;
        int iidx = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x, ++iidx) {
            const int mb = iidx % NMETA, cs = iidx % NCS;
            if (!mbar_wait(&bars->meta_full[mb], (iidx / NMETA) & 1, wc, 51))
                break;
            if (!mbar_wait(&bars->code_full[cs], (iidx / NCS) & 1, wc, 52))
                break;
            const uint32_t meta = smem_u32(sMeta + mb * meta_al);
            const uint32_t cblk = smem_u32(sCode + cs * item_code);
            for (int ks = grp; ks < KS; ks += kDnGroups) {
                uint32_t words[2][16];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int kpos = ks * kKStep + c * 32;
                    const uint4 codes = lds128(cblk + ks * kDnCodeStep + (c * kTileRows + r) * kChunkBytes);
                    if (WFMT == MOE_WFMT_Q4K) {
                        const uint4 hdr = lds128(meta + ((kpos / 256) * kTileRows + r) * 16);
                        float dsc, dm;
                        q4k_subblock_scale(hdr, (kpos % 256) / 32, dsc, dm);
                        dequant_q4k_chunk(codes, dsc, dm, words[c]);
                    } else if (WFMT == MOE_WFMT_INT4_ASYM) {
                        const uint32_t sm = lds32(meta + ((kpos >> gshift) * kTileRows + r) * 4);
                        dequant_int4asym_chunk(codes, sm, words[c]);
                    } else if (WFMT == MOE_WFMT_INT4_SYM_F16) {
                        const uint16_t sb = lds16(meta + ((kpos >> gshift) * kTileRows + r) * 2);
                        dequant_int4sym_f16_chunk(codes, sb, words[c]);
                    } else {
                        const uint16_t sb = lds16(meta + ((kpos >> gshift) * kTileRows + r) * 2);
                        dequant_int4sym_chunk(codes, sb, words[c]);
                    }
                }
                // the previous item's MMAs on this slot have finished
                if (iidx >= 1 && !mbar_wait(&bars->a_empty[ks], (iidx - 1) & 1, wc, 53)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_col = tmem + lane_off + kAccCols + ks * 32;
                tmem_st16(a_col, words[0]);
                tmem_st16(a_col + 16, words[1]);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars->a_full[ks]);
            }
            if (!ok)
                break;
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars->code_empty[cs]);
                mbar_arrive(&bars->meta_empty[mb]);
            }
        }
    } else if (warp >= 4 + kDnDeqWarps) {
        // ------------------------------------------------ epilogue (one token tile at a time)
        const int q = warp & 3;                        // TMEM lane quadrant
        const int half = (warp - 4 - kDnDeqWarps) >> 2;   // chunks half, half + 2, ...
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        uint8_t *stage = s_epi + (warp - 4 - kDnDeqWarps) * kDnEpiTok * kDnEpiStride;
        int tidx = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
            const DnItem it = dn_item<BN>(u, p, sched, n_full);
            for (int j = 0; j < it.ntiles; ++j, ++tidx) {
                const int ab = tidx & 1;
                if (!mbar_wait(&bars->acc_full[ab], (tidx >> 1) & 1, wc, 54)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int nvalid = min(BN, it.rows - j * BN);
                const int nmma = mma_width(nvalid);
                const int row0 = it.row0 + j * BN;
                const uint32_t acc = tmem + lane_off + ab * BN;
                int n0 = half * kDnEpiTok;
                uint32_t g[16], nx[16];
                if (n0 < nmma) {
                    tmem_ld16(acc + n0, g);
                    tmem_wait_ld();
                }
                for (; n0 < nmma; n0 += 2 * kDnEpiTok) {
                    // the next chunk's columns load while this one is stored
                    const bool more = n0 + 2 * kDnEpiTok < nmma;
                    if (more)
                        tmem_ld16(acc + n0 + 2 * kDnEpiTok, nx);
                    else {
                        // every column of this warp is in registers: hand the accumulator back
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0)
                            mbar_arrive(&bars->acc_empty[ab]);
                    }
                    // this lane's output feature for 16 tokens -> staging [token][feature]
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj)
                        *(__nv_bfloat16 *)(stage + jj * kDnEpiStride + lane * 2) =
                            __float2bfloat16_rn(__uint_as_float(g[jj]));
                    __syncwarp();
                    // lane: token n0 + (lane & 15), 32-byte half (lane >> 4) of the warp's 64 bytes
                    const int t = lane & 15, hh = lane >> 4;
                    const int n = n0 + t;
                    if (n < nvalid) {
                        const int prow = row0 + n;
                        uint16_t *dst = prow < p.Tk ? p.out + (size_t)prow * p.ldo
                                                    : p.out_shared + (size_t)(prow - p.Tk) * p.ldo;
                        uint4 *d4 = (uint4 *)(dst + it.f * kTileRows + q * 32 + hh * 16);
                        const uint4 *s4 = (const uint4 *)(stage + t * kDnEpiStride + hh * 32);
                        d4[0] = s4[0];
                        d4[1] = s4[1];
                    }
                    __syncwarp();
                    if (more) {
                        tmem_wait_ld();
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            g[jj] = nx[jj];
                    }
                }
                if (half * kDnEpiTok >= nmma) {
                    // no chunk of this tile for this warp
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&bars->acc_empty[ab]);
                }
            }
        }
    }

    __syncthreads();
    if (warp == 3) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

struct DnRings {
    int b_stages, b_sk, ncs, nmeta;
};

size_t dn_smem_bytes(int BN, int KS, int meta_bytes, int E_total, const DnRings &r)
{
    const size_t meta_al = (size_t)((meta_bytes + 127) & ~127);
    return 1024 + (size_t)r.b_stages * BN * 128 * r.b_sk + (size_t)r.ncs * KS * kDnCodeStep + r.nmeta * meta_al +
           sizeof(DnBars) + sizeof(int) * (32 + 4 * (size_t)E_total + 1) + 16 + kDnEpiBytes;
}

constexpr size_t kDnSmemLimit = 227 * 1024;

// B stages of four k-steps (two or one when K/64 is not a multiple of four),
// three stages where they fit, else two; two code blocks; four scale blocks
// where they fit, else two.
bool dn_rings(int BN, int KS, int meta_bytes, int E_total, DnRings &r)
{
    r.b_sk = KS % 4 == 0 ? 4 : 2;
    r.ncs = 2;
    for (r.nmeta = meta_bytes <= 4096 ? 4 : 2; r.nmeta >= 2; r.nmeta /= 2)
        for (r.b_stages = kDnMaxBStages - 1; r.b_stages >= 2; --r.b_stages)
            if (dn_smem_bytes(BN, KS, meta_bytes, E_total, r) <= kDnSmemLimit)
                return true;
    return false;
}

template <int WFMT, int BN, int SK>
cudaError_t launch_dn(const GemmArgs &a_in, int num_sms, cudaStream_t st)
{
    auto kern = down_resident_kernel<WFMT, BN, SK>;
    GemmArgs a = a_in;
    const int KS = a.K / kKStep;
    DnRings r{};
    if (!dn_rings(BN, KS, a.meta_bytes, a.E_total, r) || r.b_sk != SK)
        return cudaErrorInvalidConfiguration;
    CUtensorMap m32{}, m64{}, m128{};
    cudaError_t e = encode_kstep_map(&m32, a_in.b_src, a_in.ldb, a_in.b_rows, 32, r.b_sk);
    if (e == cudaSuccess)
        e = encode_kstep_map(&m64, a_in.b_src, a_in.ldb, a_in.b_rows, 64, r.b_sk);
    if (e == cudaSuccess)
        e = encode_kstep_map(&m128, a_in.b_src, a_in.ldb, a_in.b_rows, BN == 128 ? 128 : 64, r.b_sk);
    if (e != cudaSuccess)
        return e;
    a.b_stages = r.b_stages;
    a.b_sk = r.b_sk;
    a.ncs = r.ncs;
    a.nmeta = r.nmeta;
    const size_t smem = dn_smem_bytes(BN, KS, a.meta_bytes, a.E_total, r);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    return launch_pdl(kern, num_sms, kDnThreads, smem, st, a, m32, m64, m128);
}

}  // namespace

bool down_resident_fits(int K, int meta_bytes, int E_total)
{
    DnRings r{};
    return K % kKStep == 0 && K / kKStep <= kDnMaxKS && (K / kKStep) % 2 == 0 &&
           dn_rings(128, K / kKStep, meta_bytes, E_total, r);
}

#ifndef MOEQ4_DOWN_ITEM_TILES
#define MOEQ4_DOWN_ITEM_TILES 8
#endif

template <int SK>
cudaError_t launch_dn_fmt(const GemmArgs &a, int wfmt, int num_sms, cudaStream_t st)
{
    return wfmt == MOE_WFMT_Q4K           ? launch_dn<MOE_WFMT_Q4K, 128, SK>(a, num_sms, st)
           : wfmt == MOE_WFMT_INT4_ASYM   ? launch_dn<MOE_WFMT_INT4_ASYM, 128, SK>(a, num_sms, st)
           : wfmt == MOE_WFMT_INT4_SYM_F16 ? launch_dn<MOE_WFMT_INT4_SYM_F16, 128, SK>(a, num_sms, st)
                                           : launch_dn<MOE_WFMT_INT4_SYM, 128, SK>(a, num_sms, st);
}

cudaError_t launch_down_resident(const GemmArgs &a_in, int wfmt, int num_sms, cudaStream_t st)
{
    GemmArgs a = a_in;
    a.item_tiles = MOEQ4_DOWN_ITEM_TILES;
    const int KS = a.K / kKStep;
    if (a.item_tiles < 1 || a.item_tiles > 16 || KS > kDnMaxKS || a.K % kKStep || KS % 2)
        return cudaErrorInvalidValue;
    // k-steps per B stage: four, or two when K / 64 is not a multiple of four
    return KS % 4 == 0 ? launch_dn_fmt<4>(a, wfmt, num_sms, st) : launch_dn_fmt<2>(a, wfmt, num_sms, st);
}

}  // namespace moeq4
