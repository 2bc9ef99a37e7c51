// Kernel-side weight layout and on-chip dequantisation of 4-bit experts.
//
// Kernel layout (written by moe_pack_weights): a weight matrix set is cut
// into row tiles of 128 rows and K steps of 64.  For gate/up a tile holds
// the gate rows f*128.. and the matching up rows (NMAT = 2); for down one
// tile of Wd rows (NMAT = 1).
//   codes: per (expert, tile f, k-step ks) a contiguous block of
//          NMAT x 2 x 128 x 16 bytes, ordered [m][half c][row r]; the 16
//          bytes hold K elements ks*64 + c*32 .. +31 of row r of matrix m
//          as four 32-bit words of 8 elements: element 2i of the word in
//          nibble i, element 2i+1 in nibble i+4 (i = 0..3).  int4-sym codes
//          are stored offset-binary (q + 8), Q4K and int4-asym codes as they
//          are (0..15).
//   meta:  per (expert, tile f) a contiguous block, ordered [m][group][row]:
//          int4-sym: bf16 scale of group g (K/G groups; fp16 for the
//                    fp16-operand mode);
//          int4-asym: bf16 scale (low half) and bf16 minimum (high half);
//          Q4K:      the 16-byte super-block header (fp16 d, fp16 dmin,
//                    12 bytes of 6-bit sc/m fields) of super-block g.
// One thread owns one row and one 32-element half of a k-step, so reads of
// consecutive rows by a warp are consecutive 16-byte words.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "moeq4.h"

namespace moeq4 {

constexpr int kTileRows = 128;   // rows per tile (the MMA's M)
constexpr int kKStep = 64;       // K elements per pipeline step (one 128-byte bf16 row)
constexpr int kChunkBytes = 16;  // 32 codes

__host__ __device__ constexpr int code_block_bytes(int nmat) { return nmat * 2 * kTileRows * kChunkBytes; }

__host__ __device__ inline int meta_block_bytes(int nmat, int wfmt, int K, int G)
{
    return wfmt == MOE_WFMT_Q4K        ? nmat * (K / 256) * kTileRows * 16
           : wfmt == MOE_WFMT_INT4_ASYM ? nmat * (K / G) * kTileRows * 4
                                        : nmat * (K / G) * kTileRows * 2;   // int4-sym, bf16 or fp16 scale
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// int4-sym: 32 codes (offset-binary) and their bf16 scale -> 16 words of
// bf16 pairs, word j = elements (2j, 2j+1).  (128 + u) - 136 = q exactly;
// q * s is rounded once to bf16 (round to nearest even).
__device__ __forceinline__ void dequant_int4sym_chunk(const uint4 codes, uint16_t scale_bits, uint32_t (&out)[16])
{
    const uint32_t s2 = (uint32_t)scale_bits | ((uint32_t)scale_bits << 16);
    const uint32_t off = 0x43084308u;   // bf16 136.0 in both halves
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t t = ((w[wi] >> (4 * i)) & 0x000F000Fu) | 0x43004300u;   // bf16 pair (128+u_lo, 128+u_hi)
            out[wi * 4 + i] = bf16x2_mul(bf16x2_sub(t, off), s2);
        }
    }
}

__device__ __forceinline__ uint32_t f16x2_sub(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t f16x2_mul(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// int4-sym with an fp16 scale: 32 codes (offset-binary) -> 16 words of fp16
// pairs.  (1024 + u) - 1032 = q exactly, and q * s (at most 11 significant
// bits) is exact in fp16, so no step rounds.
__device__ __forceinline__ void dequant_int4sym_f16_chunk(const uint4 codes, uint16_t scale_bits, uint32_t (&out)[16])
{
    const uint32_t s2 = (uint32_t)scale_bits | ((uint32_t)scale_bits << 16);
    const uint32_t off = 0x64086408u;   // fp16 1032.0 in both halves
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t t = ((w[wi] >> (4 * i)) & 0x000F000Fu) | 0x64006400u;   // fp16 pair (1024+u_lo, 1024+u_hi)
            out[wi * 4 + i] = f16x2_mul(f16x2_sub(t, off), s2);
        }
    }
}

__device__ __forceinline__ float int4sym_f16_value(const uint4 codes, uint16_t scale_bits, int e)
{
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
    const int wi = e / 8, j = e % 8;
    const int nib = (j & 1) ? (j >> 1) + 4 : (j >> 1);
    const int u = (w[wi] >> (4 * nib)) & 0xF;
    return (float)(u - 8) * __half2float(__ushort_as_half(scale_bits));
}

__device__ __forceinline__ uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// int4-asym: 32 unsigned codes and the group's (scale, minimum) pair ->
// 16 words of bf16 pairs.  (128 + u) - 128 = u exactly; u * s + m is
// rounded once to bf16 by the fused multiply-add.
__device__ __forceinline__ void dequant_int4asym_chunk(const uint4 codes, uint32_t scale_min, uint32_t (&out)[16])
{
    const uint32_t s2 = __byte_perm(scale_min, 0, 0x1010);   // scale in both halves
    const uint32_t m2 = __byte_perm(scale_min, 0, 0x3232);   // minimum in both halves
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t t = ((w[wi] >> (4 * i)) & 0x000F000Fu) | 0x43004300u;   // bf16 pair (128+u_lo, 128+u_hi)
            out[wi * 4 + i] = bf16x2_fma(bf16x2_sub(t, 0x43004300u), s2, m2);
        }
    }
}

__device__ __forceinline__ float int4asym_value(const uint4 codes, uint32_t scale_min, int e)
{
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
    const int wi = e / 8, j = e % 8;
    const int nib = (j & 1) ? (j >> 1) + 4 : (j >> 1);
    const int u = (w[wi] >> (4 * nib)) & 0xF;
    const float s = __uint_as_float(scale_min << 16);
    const float m = __uint_as_float(scale_min & 0xFFFF0000u);
    return fmaf((float)u, s, m);   // u * s is exact in fp32; one rounding
}

// Exact fp32 values of the same chunk (for export): element e of 0..31.
__device__ __forceinline__ float int4sym_value(const uint4 codes, uint16_t scale_bits, int e)
{
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
    const int wi = e / 8, j = e % 8;
    const int nib = (j & 1) ? (j >> 1) + 4 : (j >> 1);
    const int u = (w[wi] >> (4 * nib)) & 0xF;
    const float s = __uint_as_float((uint32_t)scale_bits << 16);
    return (float)(u - 8) * s;
}

// Q4K super-block header -> (d*sc_j, dmin*m_j) for sub-block j, both exact in fp32.
__device__ __forceinline__ void q4k_subblock_scale(const uint4 hdr, int j, float &dsc, float &dm)
{
    const float d = __half2float(__ushort_as_half((unsigned short)(hdr.x & 0xFFFF)));
    const float dmin = __half2float(__ushort_as_half((unsigned short)(hdr.x >> 16)));
    const uint64_t lo = (uint64_t)hdr.y | ((uint64_t)hdr.z << 32);
    const uint32_t hi = hdr.w;
    auto field = [&](int f) -> uint32_t {
        const int bit = 6 * f;
        uint64_t v;
        if (bit >= 64)
            v = hi >> (bit - 64);
        else if (bit + 6 > 64)
            v = (lo >> bit) | ((uint64_t)hi << (64 - bit));
        else
            v = lo >> bit;
        return (uint32_t)(v & 63u);
    };
    dsc = d * (float)field(j);
    dm = dmin * (float)field(8 + j);
}

__device__ __forceinline__ float q4k_value_from(uint32_t u, float dsc, float dm)
{
    return fmaf(dsc, (float)u, -dm);   // d*sc*q - dmin*m, rounded once
}

// Q4K: 32 unsigned codes of one sub-block -> 16 words of bf16 pairs.
__device__ __forceinline__ void dequant_q4k_chunk(const uint4 codes, float dsc, float dm, uint32_t (&out)[16])
{
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lo = (w[wi] >> (4 * i)) & 0xFu;
            const uint32_t hi = (w[wi] >> (4 * i + 16)) & 0xFu;
            // code -> float without a conversion instruction: 2^23 + u, minus 2^23
            const float flo = __uint_as_float(0x4B000000u | lo) - 8388608.0f;
            const float fhi = __uint_as_float(0x4B000000u | hi) - 8388608.0f;
            out[wi * 4 + i] = pack_bf16x2(fmaf(dsc, flo, -dm), fmaf(dsc, fhi, -dm));
        }
    }
}

__device__ __forceinline__ float q4k_value(const uint4 codes, float dsc, float dm, int e)
{
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
    const int wi = e / 8, j = e % 8;
    const int nib = (j & 1) ? (j >> 1) + 4 : (j >> 1);
    return q4k_value_from((w[wi] >> (4 * nib)) & 0xFu, dsc, dm);
}

}  // namespace moeq4
