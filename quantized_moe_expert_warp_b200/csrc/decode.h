// Fused decode layer (decode.cu): the whole layer for T <= kDecodeMaxT tokens
// (expert intermediate I <= 1024) in one cooperative launch.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace moeq4 {

constexpr int kDecodeMaxT = 8;
constexpr int kDecodeThreads = 512;
constexpr size_t kDecodeSmemLimit = 227 * 1024;   // dynamic shared memory of one CTA

struct DecodeArgs {
    const uint16_t *x;          // [T, H] bf16
    int T, H, I, E, k, G, wfmt, renorm, has_shared;
    const float *router_w;      // [E, H]
    const float *router_bias;   // [E] or null
    const float *shared_gate;   // [H] (has_shared)
    const uint8_t *gu_q, *gu_meta, *dn_q, *dn_meta;   // kernel layout (dequant.cuh)
    int gu_meta_bytes, dn_meta_bytes;                 // per (expert, tile) meta block
    const int32_t *override_ids;   // [T, k] routing given by the caller, or null
    const float *override_w;       // [T, k]
    float *logits;              // [T, E]
    float *gate_logit;          // [T]
    int32_t *topk_ids;          // [T, k]
    float *topk_w;              // [T, k]
    uint16_t *h;                // [NP, I] gate/up outputs (bf16), NP = T k (+ T)
    uint16_t *y;                // [T, H] bf16
    int *status;                // [code, detail]
    unsigned *bar;              // [arrival word, unused, abort flag] of the grid barrier
};

// Byte offsets of the decode kernel's dynamic shared memory.
struct DecodeSmem {
    int big, red, ored, cbuf, ids, w, pidx, pair_tok, pair_w, slot_e, slot_base, slot_cnt, tcount, dexp, dbase,
        bitmap, wprefix, flag;
    int nred;     // gate/up partials buffers (1 or 2)
    int ntok;     // pairs (MMA columns) a slot holds at most: min(8, T k)
    int nstage;   // depth of each warp's staging ring
    size_t bytes;
};
DecodeSmem decode_smem_layout(int T, int k, int H, int I, int has_shared, int wfmt);
cudaError_t launch_decode_layer(const DecodeArgs &a, int grid, cudaStream_t st);

}  // namespace moeq4
