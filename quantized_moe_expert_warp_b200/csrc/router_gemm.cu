// Router logits on tcgen05 tensor cores, both operands staged by TMA.
//
// The router of the A3B layer (hipfire 0.4.3 benchmarks, "Qwen3.6-35B-A3B
// prefill on the R9700" table) scores every token against every expert:
//     logits[t, e] = x[t] . Wr[e] (+ bias[e]),  x bf16, Wr fp32.
// The fp32 weights are first split into two bf16 matrices, hi = bf16(w) and
// lo = bf16(w - hi) (w - hi is exact in fp32, and hi + lo carries 16
// significand bits of w); x is exact in bf16, so both products are exact in
// fp32 and the MMAs accumulate x.hi + x.lo in one fp32 accumulator.
//
// The GEMM is a plain warp-specialised tile loop: experts are the MMA's M =
// 128 side, tokens its N (up to 128), a k-step is 64 elements of H.  Each
// k-step stages three 128 x 64 bf16 tiles (hi, lo, x) in 128-byte swizzled
// shared memory with TMA and issues eight MMAs (hi and lo per 16 of K) from
// shared memory into a TMEM accumulator; two accumulators let the epilogue
// of one tile run under the MMAs of the next.  Small T splits H into slices
// whose partial logits are summed later (by the route kernel or the router
// reduce kernel).
//
// Warp roles of one persistent CTA (one per SM, 384 threads):
//   warp 0        TMA producer
//   warp 1        MMA issuer (one elected thread) and stage releases
//   warp 2        TMEM allocation; then shared-expert gate logits
//   warp 3        shared-expert gate logits
//   warps 4-7     epilogue (TMEM lane quadrant warp % 4)
//   warps 8-11    shared-expert gate logits
// Every wait is bounded; on timeout the CTA records MOE_ERR_TIMEOUT and
// unwinds.
#include <cstdint>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "dequant.cuh"
#include "kernels.h"
#include "moeq4.h"
#include "ptx.cuh"

namespace moeq4 {

namespace {

constexpr int kRtThreads = 384;
constexpr int kRtStages = 4;
constexpr int kRtTile = 128;                          // experts per tile (M) and tokens per tile (N)
constexpr int kRtTileBytes = kRtTile * kKStep * 2;    // one 128 x 64 bf16 tile: 16 KB
constexpr int kRtStageBytes = 3 * kRtTileBytes;       // hi, lo, x
constexpr int kRtTmemCols = 2 * kRtTile;              // two accumulators

struct RouterArgs {
    const uint16_t *x;      // [T, H] bf16 (gate logits read it directly)
    int T, H, E, E_pad;     // E_pad: rows per split matrix (a multiple of 128)
    int ksplit;             // H slices; partial s at out + s * T * E
    const float *bias;      // [E] or null (added here only without slices)
    const float *gate_w;    // [H] or null
    float *gate_out;        // [T]
    float *out;             // logits [T, E] or partials [ksplit, T, E]
    int *status;
};

struct RtBars {
    uint64_t full[kRtStages];
    uint64_t empty[kRtStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int never_abort;
};

struct RtUnit {
    int tok0, nvalid, nmma, f, split, ks0, nks;
};

// Units are ordered token tile, then expert tile, then H slice, so that the
// CTAs working at the same time share their x tiles in L2.
__device__ __forceinline__ RtUnit rt_unit(int u, const RouterArgs &p)
{
    RtUnit r;
    const int F = p.E_pad / kRtTile;
    r.split = u % p.ksplit;
    u /= p.ksplit;
    r.f = u % F;
    const int j = u / F;
    r.tok0 = j * kRtTile;
    r.nvalid = min(kRtTile, p.T - r.tok0);
    r.nmma = max(16, (r.nvalid + 15) & ~15);
    r.nks = p.H / kKStep / p.ksplit;
    r.ks0 = r.split * r.nks;
    return r;
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

// Wr [E, H] fp32 -> out [2, E_pad, H] bf16: the hi rows, then the lo rows;
// rows E .. E_pad - 1 of both are zero.  Eight weights per thread.
__global__ void __launch_bounds__(256) router_split_kernel(const float *__restrict__ w, int E, int E_pad, int H,
                                                           uint16_t *__restrict__ out)
{
    pdl_wait();
    pdl_allow_successor();
    const size_t n8 = (size_t)E_pad * H / 8;
    uint4 *hi = (uint4 *)out;
    uint4 *lo = hi + n8;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
        const size_t e = i * 8 / H;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
        if (e < (size_t)E) {
            a = *(const float4 *)(w + i * 8);
            b = *(const float4 *)(w + i * 8 + 4);
        }
        uint4 h, l;
        split2(a.x, a.y, h.x, l.x);
        split2(a.z, a.w, h.y, l.y);
        split2(b.x, b.y, h.z, l.z);
        split2(b.z, b.w, h.w, l.w);
        hi[i] = h;
        lo[i] = l;
    }
}

// gate_out[t] = x[t] . g in fp32: one warp per token, lane l takes the
// 8-element chunks l, l + 32, ... in order, then a butterfly sum over the
// lanes.  A warp takes two tokens at a time, and a token's whole row (up to
// 2048 elements: eight 16-byte loads per lane) is loaded before its FMAs.
__device__ void gate_logits(const RouterArgs &p, int worker, int nworkers)
{
    const int lane = threadIdx.x % 32;
    constexpr int kChunks = 8;   // 16-byte loads in flight per lane and token
    for (int t0 = 2 * worker; t0 < p.T; t0 += 2 * nworkers) {
        float acc[2] = {0.f, 0.f};
        for (int base = lane * 8; base < p.H; base += kChunks * 256) {
            uint4 v[2][kChunks];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int t = t0 + u;
                const uint16_t *xr = p.x + (size_t)(t < p.T ? t : t0) * p.H;
#pragma unroll
                for (int q = 0; q < kChunks; ++q)
                    v[u][q] = base + q * 256 < p.H ? *(const uint4 *)(xr + base + q * 256) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int q = 0; q < kChunks; ++q) {
                const int c0 = base + q * 256;
                if (c0 < p.H) {
                    const float4 g0 = *(const float4 *)(p.gate_w + c0);
                    const float4 g1 = *(const float4 *)(p.gate_w + c0 + 4);
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        acc[u] = fmaf(__uint_as_float(v[u][q].x << 16), g0.x, acc[u]);
                        acc[u] = fmaf(__uint_as_float(v[u][q].x & 0xFFFF0000u), g0.y, acc[u]);
                        acc[u] = fmaf(__uint_as_float(v[u][q].y << 16), g0.z, acc[u]);
                        acc[u] = fmaf(__uint_as_float(v[u][q].y & 0xFFFF0000u), g0.w, acc[u]);
                        acc[u] = fmaf(__uint_as_float(v[u][q].z << 16), g1.x, acc[u]);
                        acc[u] = fmaf(__uint_as_float(v[u][q].z & 0xFFFF0000u), g1.y, acc[u]);
                        acc[u] = fmaf(__uint_as_float(v[u][q].w << 16), g1.z, acc[u]);
                        acc[u] = fmaf(__uint_as_float(v[u][q].w & 0xFFFF0000u), g1.w, acc[u]);
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                acc[u] += __shfl_xor_sync(0xFFFFFFFFu, acc[u], off);
        }
        if (lane == 0) {
            p.gate_out[t0] = acc[0];
            if (t0 + 1 < p.T)
                p.gate_out[t0 + 1] = acc[1];
        }
    }
}

__global__ void __launch_bounds__(kRtThreads, 1)
    router_gemm_kernel(const __grid_constant__ RouterArgs p, const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ CUtensorMap tmap_x)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    RtBars *bars = (RtBars *)(smem + kRtStages * kRtStageBytes);
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRtStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
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
    pdl_wait();
    pdl_allow_successor();
    if (warp == 2) {
        tmem_alloc(&bars->tmem_base, kRtTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    const int total = ((p.T + kRtTile - 1) / kRtTile) * (p.E_pad / kRtTile) * p.ksplit;
    WaitCtx wc{&bars->abort_flag, p.status, globaltimer_ns(), wait_limit_ns(p.status)};

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (elect_one()) {
            tma_prefetch_desc(&tmap_w);
            tma_prefetch_desc(&tmap_x);
        }
        __syncwarp();
        int step = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
            const RtUnit un = rt_unit(u, p);
            for (int ks = un.ks0; ks < un.ks0 + un.nks; ++ks, ++step) {
                const int s = step % kRtStages;
                if (step >= kRtStages && !warp_wait(&bars->empty[s], ((step / kRtStages) & 1) ^ 1, wc, 31)) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    uint8_t *st = smem + s * kRtStageBytes;
                    mbar_arrive_expect_tx(&bars->full[s], (uint32_t)kRtStageBytes);
                    tma_load_2d(st, &tmap_w, ks * kKStep, un.f * kRtTile, &bars->full[s]);
                    tma_load_2d(st + kRtTileBytes, &tmap_w, ks * kKStep, p.E_pad + un.f * kRtTile, &bars->full[s]);
                    tma_load_2d(st + 2 * kRtTileBytes, &tmap_x, ks * kKStep, un.tok0, &bars->full[s]);
                }
                __syncwarp();
            }
        }
        drain_ring(bars->full, step, kRtStages, p.status, 32, &bars->never_abort);
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        int step = 0, uidx = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x, ++uidx) {
            const RtUnit un = rt_unit(u, p);
            const uint32_t idesc = idesc_bf16_f32(128, un.nmma);
            const int ab = uidx & 1;
            const uint32_t acc = tmem + ab * kRtTile;
            if (uidx >= 2) {
                if (!mbar_wait(&bars->acc_empty[ab], ((uidx >> 1) & 1) ^ 1, wc, 33))
                    break;
                tc_fence_after();
            }
            for (int ks = 0; ks < un.nks; ++ks, ++step) {
                const int s = step % kRtStages;
                if (!mbar_wait(&bars->full[s], (step / kRtStages) & 1, wc, 34)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t st = smem_u32(smem + s * kRtStageBytes);
                const uint64_t dhi = sdesc_kmajor_sw128(st);
                const uint64_t dlo = sdesc_kmajor_sw128(st + kRtTileBytes);
                const uint64_t dx = sdesc_kmajor_sw128(st + 2 * kRtTileBytes);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t adv = (uint64_t)(kk * 2);   // +32 bytes along K
                        mma_ss_f16(acc, dhi + adv, dx + adv, idesc, (ks | kk) != 0);
                        mma_ss_f16(acc, dlo + adv, dx + adv, idesc, 1);
                    }
                    mma_commit(&bars->empty[s]);
                }
                __syncwarp();
            }
            if (ok) {
                if (elect_one())
                    mma_commit(&bars->acc_full[ab]);
                __syncwarp();
            }
        }
        if (elect_one())
            mma_commit(&bars->drain);
        __syncwarp();
        WaitCtx wd{&bars->never_abort, p.status, globaltimer_ns(), kWaitLimitNs};
        warp_wait(&bars->drain, 0, wd, 35);
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------ epilogue: lane = expert, columns = tokens
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        int uidx = 0;
        for (int u = blockIdx.x; u < total; u += gridDim.x, ++uidx) {
            const RtUnit un = rt_unit(u, p);
            const int ab = uidx & 1;
            if (!mbar_wait(&bars->acc_full[ab], (uidx >> 1) & 1, wc, 36))
                break;
            tc_fence_after();
            const uint32_t acc = tmem + lane_off + ab * kRtTile;
            const int e = un.f * kRtTile + r;
            const float b = p.ksplit == 1 && p.bias && e < p.E ? p.bias[e] : 0.f;
            float *out = p.out + (size_t)un.split * p.T * p.E;
            for (int n0 = 0; n0 < un.nmma; n0 += 16) {
                uint32_t g[16];
                tmem_ld16(acc + n0, g);
                tmem_wait_ld();
                if (e < p.E) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int n = n0 + j;
                        if (n < un.nvalid)
                            out[(size_t)(un.tok0 + n) * p.E + e] = __uint_as_float(g[j]) + b;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars->acc_empty[ab]);
        }
    } else if (p.gate_w) {
        // ------------------------------------------------ shared-expert gate logits (warps 2, 3, 8-11)
        const int gw = warp < 4 ? warp - 2 : warp - 6;   // 0 .. 5
        gate_logits(p, blockIdx.x * 6 + gw, gridDim.x * 6);
    }

    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, kRtTmemCols);
    }
}

}  // namespace

// K slices of the router GEMM: enough work units (128 experts x 128 tokens x
// K slice) to cover the SMs, at most 32 slices, each a whole number of
// k-steps, and at most 4 MB of partial logits (they are written and read
// back once more).
int router_ksplit(int T, int E, int H, int sms)
{
    const int units = ((E + kRtTile - 1) / kRtTile) * ((T + 127) / 128);
    const int ks = H / kKStep;
    const size_t part_cap = (size_t)4 << 20;
    int s = 1;
    while (2 * s <= 32 && ks % (2 * s) == 0 && units * 2 * s <= sms &&
           (size_t)2 * s * T * E * sizeof(float) <= part_cap)
        s *= 2;
    return s;
}

int router_rows_padded(int E) { return (E + kRtTile - 1) / kRtTile * kRtTile; }

size_t router_split_bytes(int E, int H) { return (size_t)2 * router_rows_padded(E) * H * sizeof(uint16_t); }

cudaError_t launch_router_gemm(const uint16_t *x, int T, int H, const float *wr, const float *bias, int E,
                               const float *gate_w, float *logits, float *gate_out, int ksplit, uint16_t *wsplit,
                               int *status, int num_sms, cudaStream_t st)
{
    if (T == 0)
        return cudaSuccess;
    if (ksplit < 1 || (H / kKStep) % ksplit || H % kKStep)
        return cudaErrorInvalidValue;
    const int E_pad = router_rows_padded(E);
    cudaError_t e;
    {
        const size_t n8 = (size_t)E_pad * H / 8;
        const int blocks = (int)((n8 + 255) / 256 < 2048 ? (n8 + 255) / 256 : 2048);
        e = launch_pdl(router_split_kernel, blocks, 256, 0, st, wr, E, E_pad, H, wsplit);
        if (e != cudaSuccess)
            return e;
    }
    CUtensorMap tw{}, tx{};
    e = encode_b_map(&tw, wsplit, H, 2 * E_pad, kRtTile);
    if (e == cudaSuccess)
        e = encode_b_map(&tx, x, H, T, kRtTile);
    if (e != cudaSuccess)
        return e;
    RouterArgs a{};
    a.x = x;
    a.T = T;
    a.H = H;
    a.E = E;
    a.E_pad = E_pad;
    a.ksplit = ksplit;
    a.bias = bias;
    a.gate_w = gate_out ? gate_w : nullptr;
    a.gate_out = gate_out;
    a.out = logits;
    a.status = status;
    const size_t smem = 1024 + (size_t)kRtStages * kRtStageBytes + sizeof(RtBars);
    e = cudaFuncSetAttribute(router_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    const int units = ((T + kRtTile - 1) / kRtTile) * (E_pad / kRtTile) * ksplit;
    int grid = num_sms;
    // enough CTAs for the gate logits even when there are few GEMM units
    if (!a.gate_w && units < grid)
        grid = units;
    return launch_pdl(router_gemm_kernel, grid, kRtThreads, smem, st, a, tw, tx);
}

}  // namespace moeq4
