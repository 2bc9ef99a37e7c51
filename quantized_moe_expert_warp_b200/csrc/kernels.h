// Internal launchers shared by the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cstdlib>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

#include "moeq4.h"

namespace moeq4 {

// Launch with programmatic dependent launch: the kernel may be scheduled
// while its predecessor in the stream is still running (once every CTA of
// the predecessor has allowed it) and waits inside (griddepcontrol.wait)
// until the predecessor has finished and its writes are visible.  Every
// hot-path kernel waits before its first global read or write, so the
// ordering of the stream is unchanged; only launch latency is hidden.
// MOEQ4_NO_PDL=1 launches without it.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args)
{
    static const bool off = [] {
        const char *e = getenv("MOEQ4_NO_PDL");
        return e && e[0] == '1';
    }();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = off ? 0 : 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}


struct GemmArgs {
    const uint8_t *wq;          // codes, kernel layout
    const uint8_t *wmeta;       // scales / super-block headers, kernel layout
    const uint16_t *b_src;      // token rows of the routed experts: x in permuted order [T k, H], or h [rows, I]
    int ldb;                    // elements per row of b_src (and b_src2)
    int b_rows;                 // rows of b_src
    const uint16_t *b_src2;     // gate/up with a shared expert: its token rows x [T, H]; else null
    int b_rows2;                // rows of b_src2
    const int32_t *sorted_slot; // permutation (gather pass)
    int topk;
    int Tk;                     // T * k: rows at or past Tk belong to the shared expert
    const int32_t *offsets;     // [E + 1] permutation offsets of the routed experts
    int E;                      // routed experts
    int T;                      // tokens (rows of the shared expert)
    int E_total;                // E (+ 1 with a shared expert)
    int K;                      // reduction length (H for gate/up, I for down)
    int F;                      // 128-row tiles per expert matrix
    int G;                      // int4-sym group size
    int meta_bytes;             // per (expert, tile) meta block
    int ck_log2;                // k-steps per code chunk (set by the launcher)
    int ncs_log2;               // code chunks in the ring (set by the launcher)
    int nmeta_log2;             // meta blocks in the ring (set by the launcher)
    int item_tiles;             // resident down pass: token tiles per work item (set by the launcher)
    int b_stages, b_sk;         // resident down pass: B stages and k-steps per stage (set by the launcher)
    int ncs, nmeta;             // resident down pass: code and scale ring depths (set by the launcher)
    uint16_t *out;              // routed rows: out + p * ldo
    uint16_t *out_shared;       // shared rows: out_shared + (p - Tk) * ldo
    int ldo;
    int *status;                // [code, detail]
};

// Token-tile width of the gate/up GEMM (64, 128, 160 or 192; see gemm.cu).
int gemm_tile_tokens(int T, int E, int k, int wfmt);
// Token-tile width of the down pass: 256 when experts average >= 128 rows, else as above.
int gemm_down_tile_tokens(int T, int E, int k);
cudaError_t launch_grouped_gemm(const GemmArgs &a, int nmat, int wfmt, int tile_tokens, int num_sms, cudaStream_t st);
// Down pass with each dequantised 128-row weight tile resident in TMEM
// (K <= 512) for up to eight token tiles of 128; down_resident_fits tells
// whether a configuration can take it.
bool down_resident_fits(int K, int meta_bytes, int E_total);
cudaError_t launch_down_resident(const GemmArgs &a, int wfmt, int num_sms, cudaStream_t st);
size_t gemm_smem_required(int nmat, int meta_bytes, int E_total);

// Tensor map of a row-major 16-bit matrix [rows, ld] in boxes of 64
// elements (128 bytes, 128-byte swizzle: the MMA's K-major layout) by
// box_rows rows.
cudaError_t encode_b_map(CUtensorMap *m, const uint16_t *src, int ld, int rows, int box_rows);
// The same rows as a 3D map (64 elements, rows, ld / 64 k-steps; the third
// dimension steps 128 bytes) in boxes of box_rows rows by box_ksteps
// k-steps: one copy lands box_ksteps swizzled [box_rows x 64] slabs.
cudaError_t encode_kstep_map(CUtensorMap *m, const uint16_t *src, int ld, int rows, int box_rows, int box_ksteps);

// Router logits (or their K-slice partials) and the shared expert's gate
// logits; wsplit: router_split_bytes(E, H) of scratch for the bf16 hi/lo
// copies of the weights.  Two launches.
cudaError_t launch_router_gemm(const uint16_t *x, int T, int H, const float *wr, const float *bias, int E,
                               const float *gate_w, float *logits, float *gate_out, int ksplit, uint16_t *wsplit,
                               int *status, int num_sms, cudaStream_t st);
size_t router_split_bytes(int E, int H);
int router_ksplit(int T, int E, int H, int sms);
// Top-k routing on logits [T, E], or on the sum of `nsplit` partials
// part[s][T][E] (summed in slice order, bias added last); with partials the
// summed logits are also written to `logits` when it is not null.
cudaError_t launch_route(const float *logits, int T, int E, int k, int renorm, int32_t *ids, float *w,
                         cudaStream_t st, const float *part = nullptr, int nsplit = 1, const float *bias = nullptr,
                         float *logits_out = nullptr);
// logits = sum of the partials in slice order + bias (same order as launch_route)
cudaError_t launch_router_reduce(const float *part, int nsplit, int T, int E, const float *bias, float *logits,
                                 cudaStream_t st);

size_t permute_scratch_bytes(int T, int E, int k);
int permute_launch_count(int T, int k);   // kernels launch_permute runs
cudaError_t launch_permute(const int32_t *ids, int T, int E, int k, int32_t *counts, int32_t *offsets,
                           int32_t *sorted_slot, int32_t *dest_pos, void *scratch, int *status, cudaStream_t st);

int noalloc_max_experts();
cudaError_t launch_permute_noalloc(const int32_t *ids, int T, int E, int k, int32_t *counts, int32_t *offsets,
                                   int32_t *sorted_slot, int32_t *dest_pos, cudaStream_t st);

// out[p] = x[sorted_slot[p] / k] for p < rows, then out[rows + t] = x[t] for
// t < shared_rows (x, out: rows of H 16-bit elements).  to_f16: bf16 x is
// written as fp16, and a value beyond fp16's range records
// MOE_ERR_UNSUPPORTED (detail 40) in status.
cudaError_t launch_gather_rows(const uint16_t *x, const int32_t *sorted_slot, int rows, int k, int H, uint16_t *out,
                               int num_sms, cudaStream_t st, int shared_rows = 0, bool to_f16 = false,
                               int *status = nullptr);

cudaError_t launch_combine(const uint16_t *y_perm, const int32_t *dest_pos, const float *w, const uint16_t *shared_out,
                           const float *gate_logit, int T, int H, int k, uint16_t *y, int num_sms, cudaStream_t st);

cudaError_t launch_pack_codes(const moe_config_t &cfg, int which, const uint8_t *canon, uint8_t *out,
                              cudaStream_t st);
// fp16-operand mode: synchronises st and adds to *misfits the scales for
// which q * s would not be exact in fp16
cudaError_t launch_pack_meta(const moe_config_t &cfg, int which, const uint8_t *canon, const uint16_t *scale,
                             uint8_t *out, cudaStream_t st, unsigned *misfits = nullptr);
cudaError_t launch_dequant_export(const moe_config_t &cfg, int which, int expert, const uint8_t *q,
                                  const uint8_t *meta, float *out_f32, uint16_t *out_bf16, cudaStream_t st);

}  // namespace moeq4
