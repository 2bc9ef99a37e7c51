// Weight preparation: canonical 4-bit formats -> the GEMM kernels' layout,
// and the matching decoder used to export dequantised weights.
//
// Formats: symmetric int4 with one bf16 scale per G weights (hipfire 0.4.3
// benchmarks, "Read this before comparing columns": the mq4rs file's
// symmetric experts), asymmetric int4 with a bf16 scale and minimum per G
// weights (the same table's mq4r file), and Q4_K-style super-blocks
// (hipEngine post, "GGUF": Q4_K_S / Q4_K_M).  The pages give neither bit layout; the canonical
// layouts are described in moeq4.h, the kernel layout in dequant.cuh.
// Packing is a pure byte shuffle (plus the offset-binary flip of int4-sym
// codes); the load-time "symmetry scan" of the benchmarks page ("Other
// measured changes") corresponds to the format check done by the caller.
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "dequant.cuh"
#include "kernels.h"

namespace moeq4 {

struct MatGeom {
    int nmat, rows_per_mat, K, F, KS, rows_total, meta_bytes, ngroups;
};

static MatGeom geom(const moe_config_t &c, int which)
{
    MatGeom g;
    g.nmat = which == 0 ? 2 : 1;
    g.rows_per_mat = which == 0 ? c.I : c.H;
    g.K = which == 0 ? c.H : c.I;
    g.F = g.rows_per_mat / kTileRows;
    g.KS = g.K / kKStep;
    g.rows_total = g.nmat * g.rows_per_mat;
    g.meta_bytes = meta_block_bytes(g.nmat, c.wfmt, g.K, c.G);
    g.ngroups = c.wfmt == MOE_WFMT_Q4K ? g.K / 256 : g.K / c.G;   // int4-sym and int4-asym: K / G
    return g;
}

__device__ __forceinline__ size_t canon_row_bytes(int wfmt, int K)
{
    return wfmt == MOE_WFMT_Q4K ? (size_t)(K / 256) * 144 : (size_t)K / 2;
}

// one thread per 16-byte chunk of the kernel layout
__global__ void pack_codes_kernel(const uint8_t *__restrict__ canon, uint8_t *__restrict__ out, size_t nchunks,
                                  int wfmt, MatGeom g)
{
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= nchunks)
        return;
    size_t q = idx;
    const int r = (int)(q % kTileRows); q /= kTileRows;
    const int c = (int)(q % 2); q /= 2;
    const int m = (int)(q % g.nmat); q /= g.nmat;
    const int ks = (int)(q % g.KS); q /= g.KS;
    const int f = (int)(q % g.F); q /= g.F;
    const size_t e = q;
    const int row = m * g.rows_per_mat + f * kTileRows + r;
    const int k0 = ks * kKStep + c * 32;
    const uint8_t *src = canon + (e * g.rows_total + row) * canon_row_bytes(wfmt, g.K);
    if (wfmt == MOE_WFMT_Q4K)
        src += (size_t)(k0 / 256) * 144 + 16 + (k0 % 256) / 2;
    else
        src += k0 / 2;
    // int4-sym codes (either operand mode) become offset-binary
    const uint32_t flip = wfmt == MOE_WFMT_INT4_SYM || wfmt == MOE_WFMT_INT4_SYM_F16 ? 8u : 0u;
    uint32_t words[4];
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
        uint32_t wv = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t b = src[wi * 4 + i];
            wv |= ((b & 0xFu) ^ flip) << (4 * i);          // element 2i
            wv |= (((b >> 4) & 0xFu) ^ flip) << (4 * i + 16);  // element 2i+1
        }
        words[wi] = wv;
    }
    *(uint4 *)(out + idx * kChunkBytes) = make_uint4(words[0], words[1], words[2], words[3]);
}

// Scales of the fp16-operand mode that q * s would not be exact for, counted
// by pack_meta_kernel; read back by launch_pack_meta.
static __device__ unsigned int g_f16_scale_misfits;

// A bf16 scale as fp16 bits; *fits = false where q * s (q in [-8, 7]) would
// not be exact in fp16: s outside [2^-17, 8188] (zero allowed) or not finite.
__device__ __forceinline__ uint16_t scale_to_f16(uint16_t b, bool *fits)
{
    const float s = __uint_as_float((uint32_t)b << 16);
    const float a = fabsf(s);
    *fits = s == 0.f || (a >= 0x1p-17f && a <= 8188.f);
    return __half_as_ushort(__float2half_rn(s));
}

// int4-sym: one thread per bf16 scale (stored as fp16 in the fp16-operand
// mode); int4-asym: per (scale, minimum) pair; Q4K: per 16-byte header
__global__ void pack_meta_kernel(const uint8_t *__restrict__ canon, const uint16_t *__restrict__ scale,
                                 uint8_t *__restrict__ out, size_t n, int wfmt, int G, MatGeom g)
{
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= n)
        return;
    size_t q = idx;
    const int r = (int)(q % kTileRows); q /= kTileRows;
    const int grp = (int)(q % g.ngroups); q /= g.ngroups;
    const int m = (int)(q % g.nmat); q /= g.nmat;
    const int f = (int)(q % g.F); q /= g.F;
    const size_t e = q;
    const int row = m * g.rows_per_mat + f * kTileRows + r;
    if (wfmt == MOE_WFMT_Q4K) {
        const uint8_t *src = canon + (e * g.rows_total + row) * (size_t)(g.K / 256) * 144 + (size_t)grp * 144;
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = (uint32_t)src[4 * i] | ((uint32_t)src[4 * i + 1] << 8) | ((uint32_t)src[4 * i + 2] << 16) |
                   ((uint32_t)src[4 * i + 3] << 24);
        *(uint4 *)(out + idx * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    } else if (wfmt == MOE_WFMT_INT4_ASYM) {
        const size_t i = ((e * g.rows_total + row) * (size_t)(g.K / G) + grp) * 2;
        ((uint32_t *)out)[idx] = (uint32_t)scale[i] | ((uint32_t)scale[i + 1] << 16);
    } else if (wfmt == MOE_WFMT_INT4_SYM_F16) {
        bool fits;
        ((uint16_t *)out)[idx] = scale_to_f16(scale[(e * g.rows_total + row) * (size_t)(g.K / G) + grp], &fits);
        if (!fits)
            atomicAdd(&g_f16_scale_misfits, 1u);
    } else {
        ((uint16_t *)out)[idx] = scale[(e * g.rows_total + row) * (size_t)(g.K / G) + grp];
    }
}

cudaError_t launch_pack_codes(const moe_config_t &cfg, int which, const uint8_t *canon, uint8_t *out,
                              cudaStream_t st)
{
    const MatGeom g = geom(cfg, which);
    const size_t E_total = (size_t)cfg.E + (cfg.has_shared ? 1 : 0);
    const size_t n = E_total * g.F * g.KS * g.nmat * 2 * kTileRows;
    pack_codes_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(canon, out, n, cfg.wfmt, g);
    return cudaGetLastError();
}

cudaError_t launch_pack_meta(const moe_config_t &cfg, int which, const uint8_t *canon, const uint16_t *scale,
                             uint8_t *out, cudaStream_t st, unsigned *misfits)
{
    const MatGeom g = geom(cfg, which);
    const size_t E_total = (size_t)cfg.E + (cfg.has_shared ? 1 : 0);
    const size_t n = E_total * g.F * g.nmat * g.ngroups * kTileRows;
    void *counter = nullptr;
    cudaError_t e = cudaSuccess;
    if (cfg.wfmt == MOE_WFMT_INT4_SYM_F16) {
        // the count lives in this library's device memory: its address is
        // looked up on the current device (set-up path, not stream work)
        e = cudaGetSymbolAddress(&counter, g_f16_scale_misfits);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(counter, 0, sizeof(unsigned), st);
        if (e != cudaSuccess)
            return e;
    }
    pack_meta_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(canon, scale, out, n, cfg.wfmt, cfg.G, g);
    e = cudaGetLastError();
    if (e == cudaSuccess && counter) {
        unsigned host = 0;
        e = cudaMemcpyAsync(&host, counter, sizeof(unsigned), cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess)
            e = cudaStreamSynchronize(st);
        if (misfits)
            *misfits += host;
    }
    return e;
}

// one thread per (row, 32-element chunk) of one expert matrix
__global__ void dequant_export_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ meta, int e, int wfmt,
                                      int G, MatGeom g, float *out_f32, uint16_t *out_bf16)
{
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    const int nk = g.K / 32;
    if (idx >= g.rows_total * nk)
        return;
    const int R = idx / nk, kc = idx % nk;
    const int m = R / g.rows_per_mat, rr = R % g.rows_per_mat;
    const int f = rr / kTileRows, r = rr % kTileRows;
    const int ks = kc / 2, c = kc % 2;
    const size_t tile = (size_t)e * g.F + f;
    const uint4 codes =
        *(const uint4 *)(q + ((((tile * g.KS + ks) * g.nmat + m) * 2 + c) * kTileRows + r) * kChunkBytes);
    const uint8_t *mb = meta + tile * g.meta_bytes;
    const int kpos = kc * 32;
    uint32_t words[16];
    float vals[32];
    if (wfmt == MOE_WFMT_Q4K) {
        const int sb = kpos / 256;
        const uint4 hdr = *(const uint4 *)(mb + ((m * g.ngroups + sb) * kTileRows + r) * 16);
        float dsc, dm;
        q4k_subblock_scale(hdr, (kpos % 256) / 32, dsc, dm);
        dequant_q4k_chunk(codes, dsc, dm, words);
        for (int i = 0; i < 32; ++i)
            vals[i] = q4k_value(codes, dsc, dm, i);
    } else if (wfmt == MOE_WFMT_INT4_ASYM) {
        const int grp = kpos / G;
        const uint32_t sm = *(const uint32_t *)(mb + ((m * g.ngroups + grp) * kTileRows + r) * 4);
        dequant_int4asym_chunk(codes, sm, words);
        for (int i = 0; i < 32; ++i)
            vals[i] = int4asym_value(codes, sm, i);
    } else if (wfmt == MOE_WFMT_INT4_SYM_F16) {
        const int grp = kpos / G;
        const uint16_t sbits = *(const uint16_t *)(mb + ((m * g.ngroups + grp) * kTileRows + r) * 2);
        dequant_int4sym_f16_chunk(codes, sbits, words);
        for (int i = 0; i < 32; ++i)
            vals[i] = int4sym_f16_value(codes, sbits, i);
    } else {
        const int grp = kpos / G;
        const uint16_t sbits = *(const uint16_t *)(mb + ((m * g.ngroups + grp) * kTileRows + r) * 2);
        dequant_int4sym_chunk(codes, sbits, words);
        for (int i = 0; i < 32; ++i)
            vals[i] = int4sym_value(codes, sbits, i);
    }
    for (int i = 0; i < 32; ++i) {
        if (out_f32)
            out_f32[(size_t)R * g.K + kpos + i] = vals[i];
        if (out_bf16)
            out_bf16[(size_t)R * g.K + kpos + i] = (uint16_t)(i & 1 ? words[i / 2] >> 16 : words[i / 2] & 0xFFFF);
    }
}

cudaError_t launch_dequant_export(const moe_config_t &cfg, int which, int expert, const uint8_t *q,
                                  const uint8_t *meta, float *out_f32, uint16_t *out_bf16, cudaStream_t st)
{
    const MatGeom g = geom(cfg, which);
    const int n = g.rows_total * (g.K / 32);
    dequant_export_kernel<<<(n + 127) / 128, 128, 0, st>>>(q, meta, expert, cfg.wfmt, cfg.G, g, out_f32, out_bf16);
    return cudaGetLastError();
}

}  // namespace moeq4
