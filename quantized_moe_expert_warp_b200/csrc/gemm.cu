// Grouped expert GEMMs on 4-bit weights, tcgen05 tensor cores.
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
// Warp roles of one persistent CTA (one per SM, 512 threads):
//   warp 0      gathers token rows of B with cp.async (zero rows past the tail)
//   warp 1      issues tcgen05.mma (one thread) and commits stage releases
//   warp 2      streams code blocks and per-tile scale blocks with bulk copies
//   warp 3      owns the TMEM allocation
//   warps 4-11  dequantise: row r = 32*(warp%4) + lane, half c = (warp-4)/4
//   warps 12-15 epilogue (TMEM -> registers -> global)
// Every wait is bounded; on timeout the CTA records MOE_ERR_TIMEOUT and
// unwinds.
#include <cstdint>
#include <cuda_runtime.h>

#include "dequant.cuh"
#include "moeq4.h"
#include "ptx.cuh"
#include "kernels.h"

namespace moeq4 {

constexpr int kBN = 128;           // max tokens per tile (the MMA's N)
constexpr int kStages = 4;         // B / TMEM-A pipeline depth
constexpr int kThreads = 512;
constexpr int kLag = kStages - 1;  // cp.async groups in flight before a stage is signalled

template <int NMAT>
struct GemmSmem {
    static constexpr int kCodeStages = NMAT == 2 ? 8 : 16;
    static constexpr int kBBytes = kStages * kBN * 128;
    static constexpr int kCodeBytes = kCodeStages * code_block_bytes(NMAT);
    static constexpr int kTmemCols = NMAT == 2 ? 512 : 256;
    static constexpr int kAccCols = NMAT * kBN;
    // A stages follow the accumulators in TMEM
    static_assert(kAccCols + kStages * NMAT * 32 <= kTmemCols, "TMEM budget");
};

struct Barriers {
    uint64_t b_full[kStages];
    uint64_t a_full[kStages];
    uint64_t mma_done[kStages];
    uint64_t code_full[16];
    uint64_t code_empty[16];
    uint64_t meta_full[2];
    uint64_t meta_empty[2];
    uint64_t acc_full;
    uint64_t acc_empty;
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

struct Unit {
    int e, f, row0, nvalid, nmma;
};

struct Sched {
    const int *tile_start;   // [E_total + 1] first tile of each expert
    const int *row_start;    // [E_total] first permuted row
    const int *row_count;    // [E_total] rows
};

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
    r.row0 = sc.row_start[lo] + c * kBN;
    r.nvalid = min(kBN, sc.row_count[lo] - c * kBN);
    r.nmma = max(16, (r.nvalid + 15) & ~15);
    return r;
}

// Every CTA derives the tile schedule from the permutation offsets: rows of
// expert e are [offsets[e], offsets[e+1]); the shared expert (if any) is
// expert E with rows [T k, T k + T); expert e owns ceil(rows / kBN) tiles.
__device__ void build_schedule(const GemmArgs &p, int *s_tile_start, int *s_row_start, int *s_row_count,
                               int *s_part)
{
    const int n = p.E_total;
    const int per = (n + kThreads - 1) / kThreads;
    const int e0 = threadIdx.x * per;
    int local = 0;
    for (int e = e0; e < min(n, e0 + per); ++e) {
        const int start = e < p.E ? p.offsets[e] : p.Tk;
        const int cnt = e < p.E ? p.offsets[e + 1] - p.offsets[e] : p.T;
        s_row_start[e] = start;
        s_row_count[e] = cnt;
        local += (cnt + kBN - 1) / kBN;
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
        run += (s_row_count[e] + kBN - 1) / kBN;
    }
    if (threadIdx.x == kThreads - 1)
        s_tile_start[n] = s_part[kThreads - 1];
}

template <int NMAT, int WFMT, bool GATHER>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_q4_kernel(const GemmArgs p)
{
    using L = GemmSmem<NMAT>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the swizzled B stages
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sB = smem;
    uint8_t *sCode = sB + L::kBBytes;
    uint8_t *sMeta = sCode + L::kCodeBytes;
    const int meta_bytes = p.meta_bytes;
    Barriers *bars = (Barriers *)(sMeta + 2 * ((meta_bytes + 127) & ~127));
    int *s_tile_start = (int *)(bars + 1);
    int *s_row_start = s_tile_start + p.E_total + 1;
    int *s_row_count = s_row_start + p.E_total;
    int *s_part = s_row_count + p.E_total;
    const Sched sched{s_tile_start, s_row_start, s_row_count};

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->b_full[s], 1);
            mbar_init(&bars->a_full[s], 8);
            mbar_init(&bars->mma_done[s], 1);
        }
        for (int s = 0; s < L::kCodeStages; ++s) {
            mbar_init(&bars->code_full[s], 1);
            mbar_init(&bars->code_empty[s], 8);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->meta_full[s], 1);
            mbar_init(&bars->meta_empty[s], 8);
        }
        mbar_init(&bars->acc_full, 1);
        mbar_init(&bars->acc_empty, 4);
        mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    build_schedule(p, s_tile_start, s_row_start, s_row_count, s_part);
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
            const Unit un = decode_unit(u, p, sched);
            const uint16_t *src[kBN / 32];
            uint32_t bytes[kBN / 32];
#pragma unroll
            for (int i = 0; i < kBN / 32; ++i) {
                const int r = lane + 32 * i;
                const int prow = un.row0 + r;
                int srow = 0;
                if (r < un.nvalid)
                    srow = GATHER ? (prow < p.Tk ? p.sorted_slot[prow] / p.topk : prow - p.Tk) : prow;
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
                cp_async_commit();
                if (step >= kLag) {
                    cp_async_wait_group<kLag>();
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&bars->b_full[(step - kLag) % kStages]);
                }
            }
        }
        cp_async_wait_group<0>();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0)
            for (int s = max(0, step - kLag); s < step; ++s)
                mbar_arrive(&bars->b_full[s % kStages]);
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int step = 0, uidx = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++uidx) {
                const Unit un = decode_unit(u, p, sched);
                const uint32_t idesc = idesc_bf16_f32(128, un.nmma);
                if (uidx > 0) {
                    if (!mbar_wait(&bars->acc_empty, (uidx - 1) & 1, wc, 2))
                        break;
                    tc_fence_after();
                }
                for (int ks = 0; ks < KS; ++ks, ++step) {
                    const int s = step % kStages;
                    const uint32_t ph = (step / kStages) & 1;
                    if (!mbar_wait(&bars->a_full[s], ph, wc, 3) || !mbar_wait(&bars->b_full[s], ph, wc, 4)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t bbase = smem_u32(sB + s * kBN * 128);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bdesc = sdesc_kmajor_sw128(bbase + kk * 32);
#pragma unroll
                        for (int m = 0; m < NMAT; ++m) {
                            const uint32_t a_t = tmem + L::kAccCols + (s * NMAT + m) * 32 + kk * 8;
                            mma_ts_f16(tmem + m * kBN, a_t, bdesc, idesc, (ks | kk) != 0);
                        }
                    }
                    mma_commit(&bars->mma_done[s]);
                }
                if (ok)
                    mma_commit(&bars->acc_full);
            }
            // all issued MMAs finish before the CTA may release TMEM
            mma_commit(&bars->drain);
            WaitCtx wd{&bars->abort_flag, p.status, globaltimer_ns()};
            int zero = 0;
            wd.abort_flag = &zero;   // wait for the drain even after an abort
            mbar_wait(&bars->drain, 0, wd, 5);
        }
    } else if (warp == 2) {
        // ------------------------------------------------ code / meta producer
        if (lane == 0) {
            int step = 0, munit = 0;
            const int cbytes = code_block_bytes(NMAT);
            bool ok = true;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++munit) {
                const Unit un = decode_unit(u, p, sched);
                const size_t tile_id = (size_t)un.e * p.F + un.f;
                const int mb = munit & 1;
                if (munit >= 2 && !mbar_wait(&bars->meta_empty[mb], ((munit >> 1) & 1) ^ 1, wc, 6))
                    break;
                mbar_arrive_expect_tx(&bars->meta_full[mb], meta_bytes);
                bulk_g2s(sMeta + mb * ((meta_bytes + 127) & ~127), p.wmeta + tile_id * meta_bytes, meta_bytes,
                         &bars->meta_full[mb]);
                for (int ks = 0; ks < KS; ++ks, ++step) {
                    const int s = step % L::kCodeStages;
                    if (step >= L::kCodeStages &&
                        !mbar_wait(&bars->code_empty[s], ((step / L::kCodeStages) & 1) ^ 1, wc, 7)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->code_full[s], cbytes);
                    bulk_g2s(sCode + s * cbytes, p.wq + (tile_id * KS + ks) * cbytes, cbytes, &bars->code_full[s]);
                }
            }
        }
    } else if (warp >= 4 && warp < 12) {
        // ------------------------------------------------ dequant into TMEM
        const int c = (warp - 4) >> 2;            // which 32-element half of the k-step
        const int r = (warp & 3) * 32 + lane;     // tile row == TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const int cbytes = code_block_bytes(NMAT);
        int step = 0, munit = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++munit) {
            const int mb = munit & 1;
            if (!mbar_wait(&bars->meta_full[mb], (munit >> 1) & 1, wc, 8))
                break;
            const uint8_t *meta = sMeta + mb * ((meta_bytes + 127) & ~127);
            const int ngroups = WFMT == MOE_WFMT_Q4K ? p.K / 256 : p.K / p.G;
            for (int ks = 0; ks < KS; ++ks, ++step) {
                const int sc = step % L::kCodeStages;
                if (!mbar_wait(&bars->code_full[sc], (step / L::kCodeStages) & 1, wc, 9)) {
                    ok = false;
                    break;
                }
                const int kpos = ks * kKStep + c * 32;
                uint32_t words[NMAT][16];
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    const uint4 codes =
                        *(const uint4 *)(sCode + sc * cbytes + ((m * 2 + c) * kTileRows + r) * kChunkBytes);
                    if (WFMT == MOE_WFMT_Q4K) {
                        const int g = kpos / 256;
                        const uint4 hdr = *(const uint4 *)(meta + ((m * ngroups + g) * kTileRows + r) * 16);
                        float dsc, dm;
                        q4k_subblock_scale(hdr, (kpos % 256) / 32, dsc, dm);
                        dequant_q4k_chunk(codes, dsc, dm, words[m]);
                    } else {
                        const int g = kpos / p.G;
                        const uint16_t sbits = *(const uint16_t *)(meta + ((m * ngroups + g) * kTileRows + r) * 2);
                        dequant_int4sym_chunk(codes, sbits, words[m]);
                    }
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars->code_empty[sc]);
                const int sa = step % kStages;
                if (step >= kStages && !mbar_wait(&bars->mma_done[sa], ((step / kStages) & 1) ^ 1, wc, 10)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int m = 0; m < NMAT; ++m)
                    tmem_st16(tmem + lane_off + L::kAccCols + (sa * NMAT + m) * 32 + c * 16, words[m]);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars->a_full[sa]);
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars->meta_empty[mb]);
        }
    } else if (warp >= 12) {
        // ------------------------------------------------ epilogue
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        int uidx = 0;
        for (int u = blockIdx.x; u < total_units; u += gridDim.x, ++uidx) {
            const Unit un = decode_unit(u, p, sched);
            if (!mbar_wait(&bars->acc_full, uidx & 1, wc, 11))
                break;
            tc_fence_after();
            const int col = un.f * kTileRows + r;
            for (int n0 = 0; n0 < un.nmma; n0 += 16) {
                uint32_t g[16], v[16];
                tmem_ld16(tmem + lane_off + n0, g);
                if (NMAT == 2)
                    tmem_ld16(tmem + lane_off + kBN + n0, v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int n = n0 + j;
                    if (n < un.nvalid) {
                        const int prow = un.row0 + n;
                        float o;
                        if (NMAT == 2) {
                            const float a = __uint_as_float(g[j]);
                            o = a / (1.0f + __expf(-a)) * __uint_as_float(v[j]);
                        } else {
                            o = __uint_as_float(g[j]);
                        }
                        uint16_t *dst = prow < p.Tk ? p.out + (size_t)prow * p.ldo
                                                    : p.out_shared + (size_t)(prow - p.Tk) * p.ldo;
                        dst[col] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars->acc_empty);
        }
    }

    __syncthreads();
    if (warp == 3) {
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
    }
}

template <int NMAT>
static size_t gemm_smem_bytes(int meta_bytes, int E_total)
{
    using L = GemmSmem<NMAT>;
    return 1024 + L::kBBytes + L::kCodeBytes + 2 * ((meta_bytes + 127) & ~127) + sizeof(Barriers) +
           sizeof(int) * (3 * E_total + 1 + kThreads) + 16;
}

template <int NMAT, int WFMT, bool GATHER>
static cudaError_t launch_one(const GemmArgs &a, int num_sms, cudaStream_t st)
{
    auto kern = grouped_gemm_q4_kernel<NMAT, WFMT, GATHER>;
    const size_t smem = gemm_smem_bytes<NMAT>(a.meta_bytes, a.E_total);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    kern<<<num_sms, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

size_t gemm_smem_required(int nmat, int meta_bytes, int E_total)
{
    return nmat == 2 ? gemm_smem_bytes<2>(meta_bytes, E_total) : gemm_smem_bytes<1>(meta_bytes, E_total);
}

cudaError_t launch_grouped_gemm(const GemmArgs &a, int nmat, int wfmt, int num_sms, cudaStream_t st)
{
    if (nmat == 2) {
        return wfmt == MOE_WFMT_Q4K ? launch_one<2, MOE_WFMT_Q4K, true>(a, num_sms, st)
                                    : launch_one<2, MOE_WFMT_INT4_SYM, true>(a, num_sms, st);
    }
    return wfmt == MOE_WFMT_Q4K ? launch_one<1, MOE_WFMT_Q4K, false>(a, num_sms, st)
                                : launch_one<1, MOE_WFMT_INT4_SYM, false>(a, num_sms, st);
}

}  // namespace moeq4
