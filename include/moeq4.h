/*
 * moeq4 -- C ABI of the 4-bit weight-quantized Mixture-of-Experts FFN layer
 * for NVIDIA B200 (sm_100a).  Library: libmoeq4.so.
 *
 * The layer is the routed-expert FFN of a Qwen3.6-35B-A3B-style model, the
 * model the hipfire 0.4.3 benchmarks page measures ("Qwen3.6-35B-A3B
 * prefill on the R9700" table; its "Read this before comparing columns"
 * table names the MoE prefill routes: per-expert buffers, and the
 * symmetric IU4 MoE route for files with symmetric int4 experts).  The
 * hipEngine post ("GGUF" section) adds the Q4_K super-block format.  The
 * pages give no equations; the layer computed here is the plain reading:
 *
 *   logits[t,e] = x[t,:] . Wr[e,:] + bias[e]                (moe_router_logits)
 *   ids[t,:]    = the k largest logits, ties to the lower id, descending
 *   w[t,j]      = exp(L[ids[t,j]] - L_max) / sum_{i<k} exp(L[ids[t,i]] - L_max)
 *                 (renorm = 1; renorm = 0 divides by the sum over all E) (moe_route)
 *   slots s = t*k + j are sorted by expert, stably in s        (moe_permute)
 *   Y[p] = (silu(x[t_p] Wg_e^T) * (x[t_p] Wu_e^T)) Wd_e^T      (moe_expert_ffn_q4)
 *   y[t] = sum_j w[t,j] Y[dest_pos[t*k+j]] + sigmoid(x[t].g) S[t]  (moe_combine)
 *
 * where S is the same FFN with the shared expert's weights on every token.
 * moe_layer_forward runs all steps in order on one stream.
 *
 * Conventions for every call:
 *  - Returns MOE_OK (0) or a negative MOE_ERR_* code; moe_last_error()
 *    then gives a message (thread-local, valid until the next call).
 *  - Tensor pointers are DEVICE pointers owned by the caller; arrays are
 *    row-major and contiguous.  Pointers handed to kernels must be 16-byte
 *    aligned (MOE_ERR_INVALID_ARG otherwise).  The library never
 *    allocates device memory; scratch comes from a caller workspace whose
 *    size a *_workspace_size call returns.
 *  - `stream` is a cudaStream_t (NULL: the legacy default stream).  Calls
 *    enqueue kernels and return without synchronising.  Failures detected
 *    inside kernels (a wait that exceeded its time budget) are recorded in
 *    a status word inside the workspace; moe_read_status() reads it.
 *  - bf16 tensors are passed as uint16_t bit patterns.
 */
#ifndef MOEQ4_H
#define MOEQ4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1) /* null / misaligned pointer, bad size                  */
#define MOE_ERR_UNSUPPORTED (-2) /* shape or format the kernels do not admit              */
#define MOE_ERR_CUDA (-3)        /* a CUDA runtime call failed (message has the cause)    */
#define MOE_ERR_TIMEOUT (-4)     /* a device-side wait ran out of its budget               */
#define MOE_ERR_WORKSPACE (-5)   /* workspace missing or smaller than required            */

/* Expert weight formats. */
#define MOE_WFMT_INT4_SYM 0 /* int4 two's complement, one bf16 scale per G weights along K */
#define MOE_WFMT_Q4K 1      /* Q4_K-style 256-weight super-blocks (see moe_pack_weights)   */
#define MOE_WFMT_INT4_ASYM 2 /* unsigned int4, a bf16 scale and a bf16 minimum per G weights */
/* The int4-sym weights above (same canonical input), computed with fp16
 * tensor-core operands: q*s has at most 11 significant bits, so every
 * dequantised weight is exact in fp16 (scales in [2^-17, 8188], checked
 * by moe_pack_weights); the activations x enter as fp16 (exact for bf16
 * values with 2^-17 <= |x| <= 65504; smaller ones are rounded, within
 * 2^-25; larger ones are refused at run time), and the SwiGLU output h
 * is kept in fp16.  This is the library's own exact-weight route for the
 * symmetric experts (the pages' late-prefill steps on the mq4rs file keep
 * their routes byte-exact: hipfire 0.4.3 benchmarks, "Late prefill steps
 * on mq4rs"; an F16 operand route appears there for another model's 6-bit
 * file, in the Flash-Next prefill table). */
#define MOE_WFMT_INT4_SYM_F16 3

/* Shapes of one layer.  Admitted: H % 128 == 0, I % 128 == 0, 1 <= k <= E <= 1024,
 * int4-sym / int4-asym: G a power of two, G >= 32, G divides H and I; Q4K: H % 256 == 0,
 * I % 256 == 0. */
typedef struct moe_config {
    int32_t H;          /* hidden size                                   */
    int32_t I;          /* expert intermediate size (shared expert too)  */
    int32_t E;          /* routed experts                                */
    int32_t k;          /* experts per token                             */
    int32_t G;          /* int4 group size along K (ignored for Q4K)     */
    int32_t has_shared; /* 1: one always-on shared expert                */
    int32_t renorm;     /* 1: renormalise the top-k weights to sum to 1  */
    int32_t wfmt;       /* MOE_WFMT_*                                    */
} moe_config_t;

/* Device pointers of one layer's weights (caller-owned). */
typedef struct moe_layer {
    moe_config_t cfg;
    const float *router_w;    /* [E, H] fp32                                     */
    const float *router_bias; /* [E] fp32 or NULL                                */
    const float *shared_gate; /* [H] fp32 (required when has_shared)             */
    const void *gu_q;         /* gate/up codes in the kernel layout (moe_pack_weights) */
    const void *gu_meta;      /* gate/up scales or super-block headers           */
    const void *dn_q;         /* down codes in the kernel layout                 */
    const void *dn_meta;      /* down scales or super-block headers              */
} moe_layer_t;

/* Optional exports / overrides of moe_layer_forward (all device pointers,
 * each may be NULL).  When override_ids is set, routing is skipped and
 * override_ids / override_w [T, k] are used instead. */
typedef struct moe_debug {
    float *logits;            /* [T, E]  */
    float *gate_logit;        /* [T]     */
    int32_t *topk_ids;        /* [T, k]  */
    float *topk_w;            /* [T, k]  */
    int32_t *counts;          /* [E]     */
    int32_t *offsets;         /* [E + 1] */
    int32_t *sorted_slot;     /* [T k]   */
    int32_t *dest_pos;        /* [T k]   */
    const int32_t *override_ids;
    const float *override_w;
} moe_debug_t;

/* Message of the last failed call on this thread ("" if none). */
const char *moe_last_error(void);

/* ABI version (increments on incompatible change). */
int moe_version(void);

/* Number of kernels this library has enqueued in this process (host-side count). */
uint64_t moe_kernel_launches(void);

/* --------------------------------------------------------------- weights */

/* Bytes of the four kernel-layout buffers for all E (+1 shared) experts.
 * Returns MOE_ERR_UNSUPPORTED for shapes the kernels do not admit. */
int moe_packed_sizes(const moe_config_t *cfg, size_t *gu_q_bytes, size_t *gu_meta_bytes, size_t *dn_q_bytes,
                     size_t *dn_meta_bytes);

/*
 * Convert canonical expert weights (device memory) to the kernel layout.
 * Canonical, per expert e in [0, E + has_shared) (the shared expert last):
 *   gate/up matrix [2I, H] (gate rows first), down matrix [H, I];
 *   int4-sym: codes uint8 [rows, K/2] (element 2i in the low nibble,
 *             two's complement) and scales bf16 [rows, K/G];
 *   Q4K:      uint8 [rows, K/256 * 144] super-blocks: fp16 d, fp16 dmin,
 *             12 bytes of sixteen 6-bit fields (little-endian bit stream:
 *             sc_0..7 then m_0..7), 128 bytes of unsigned 4-bit q (weight
 *             i in byte i/2, low nibble when i is even);
 *             w = d*sc_j*q - dmin*m_j for sub-block j = i / 32.
 *   int4-asym: codes uint8 [rows, K/2] (unsigned q, element 2i in the low
 *             nibble) and, per group, the bf16 pair (scale s, minimum m):
 *             uint16 [rows, K/G, 2]; w = q*s + m (the pages' asymmetric
 *             mq4r file; the recipe is this library's reading);
 *   gu_scale / dn_scale are ignored (may be NULL) for Q4K.
 *   int4-sym-f16: the int4-sym input; the scales are stored as fp16.
 *             The call then synchronises `stream` and returns
 *             MOE_ERR_UNSUPPORTED if a scale lies outside [2^-17, 8188]
 *             (or is not finite), where q*s would not be exact in fp16;
 *             zero scales are accepted.
 * Outputs go to caller buffers of the sizes moe_packed_sizes() returns.
 * Source: hipfire 0.4.3 benchmarks, "Read this before comparing columns"
 * (symmetric-expert mq4rs file); hipEngine post, "GGUF" (Q4_K).  The bit
 * layouts are this library's own; the pages give none.
 */
int moe_pack_weights(const moe_config_t *cfg, const void *gu_canon, const void *gu_scale, const void *dn_canon,
                     const void *dn_scale, void *gu_q, void *gu_meta, void *dn_q, void *dn_meta, void *stream);

/*
 * Dequantised weights of one matrix of one expert, decoded from the kernel
 * layout exactly as the GEMM kernels decode them.  which = 0: gate/up
 * [2I, H]; which = 1: down [H, I].  out_f32 gets the exact values (fp32),
 * out_bf16 (optional) the bf16 operand the tensor cores consume.
 */
int moe_dequant_export(const moe_config_t *cfg, const void *q, const void *meta, int which, int expert,
                       float *out_f32, uint16_t *out_bf16, void *stream);

/* ------------------------------------------------------------ the steps */

/* Workspace bytes of moe_router_logits for up to T tokens. */
size_t moe_router_workspace_size(const moe_config_t *cfg, int T);

/*
 * Router logits and the shared expert's gate logit.
 *   x [T, H] bf16, logits [T, E] fp32 (bias added when L->router_bias),
 *   gate_logit [T] fp32 = x . shared_gate (may be NULL; ignored without a
 *   shared expert).  fp32 accumulation.  The caller's workspace ws (at
 *   least moe_router_workspace_size bytes, 256-byte aligned;
 *   MOE_ERR_WORKSPACE if smaller) receives the router weights split into
 *   two bf16 matrices (hi = bf16(w), lo = bf16(w - hi); rewritten by every
 *   call) and, for small T, the partial logits of the slices of H that run
 *   on separate SMs, summed in slice order.
 * Source: the router of the Qwen3.6-35B-A3B layer the hipfire 0.4.3
 * benchmarks measure ("Qwen3.6-35B-A3B prefill on the R9700" table); the
 * pages give no formula, so logits = x Wr^T + bias is this library's reading.
 */
int moe_router_logits(const moe_layer_t *L, const uint16_t *x, int T, float *logits, float *gate_logit, void *ws,
                      size_t ws_bytes, void *stream);

/*
 * Top-k routing, one warp per token.  logits [T, E] fp32 (finite),
 * topk_ids [T, k] int32 (descending logit, ties to the lower id),
 * topk_w [T, k] fp32.  1 <= k <= min(E, 32), E <= 1024.  A position that
 * cannot be filled because the remaining logits are NaN gets id -1 and
 * weight 0 (moe_permute then reports the id as out of range).
 * Source: the top-8 expert choice of the A3B layer (hipfire 0.4.3
 * benchmarks, "Qwen3.6-35B-A3B prefill on the R9700" table); the tie rule
 * and the renormalised softmax are this library's reading, the pages give
 * neither.
 */
int moe_route(const float *logits, int T, int E, int k, int renorm, int32_t *topk_ids, float *topk_w,
              void *stream);

/* Workspace bytes of moe_permute for T tokens. */
size_t moe_permute_workspace_size(int T, int E, int k);

/*
 * Stable counting sort of the T*k slots by expert.
 *   counts [E], offsets [E + 1] (offsets[E] = T k), sorted_slot [T k]
 *   (slot t*k + j at position p), dest_pos [T k] (inverse).  Ids outside
 *   [0, E) are a device error (status word).  ws: moe_permute_workspace_size.
 * Source: hipfire 0.4.3 benchmarks, "Read this before comparing columns"
 * table, row "MoE prefill route" (per-expert buffers): the tokens of each
 * expert gathered together; here one permutation replaces the buffers.
 */
int moe_permute(const int32_t *topk_ids, int T, int E, int k, int32_t *counts, int32_t *offsets,
                int32_t *sorted_slot, int32_t *dest_pos, void *ws, size_t ws_bytes, void *stream);

/*
 * moe_permute without a workspace, for callers that cannot allocate device
 * memory when they route (for instance code that runs under another
 * allocator's lock, or a host framework that forbids cudaMalloc after
 * start-up and hands out no scratch).  The pages have no counterpart of
 * this call; it exists for such integrations.
 *  - Same inputs, outputs and results as moe_permute (bit for bit).
 *  - Scratch: one fixed array inside the library, in device global memory,
 *    sized for E <= 1024 experts (any T); each GPU that loads the library
 *    keeps it (128 KB) until the process exits.  E > 1024 returns
 *    MOE_ERR_UNSUPPORTED.  The call allocates nothing.
 *  - The call runs on the current device, and `stream` must belong to it
 *    (otherwise MOE_ERR_INVALID_ARG).  The first call on a device looks up
 *    the array's device address for that device (a runtime call, no stream
 *    work) and keeps it; make that first call before any stream capture.
 *  - All calls on a device share the array: calls that may overlap on the GPU
 *    (unordered streams) race and must be serialised by the caller.  Nothing
 *    needs clearing between calls.
 *  - Ids outside [0, E) are not reported through a status word (there is no
 *    workspace); their dest_pos entries come back as -1.
 */
int moe_permute_noalloc(const int32_t *topk_ids, int T, int E, int k, int32_t *counts, int32_t *offsets,
                        int32_t *sorted_slot, int32_t *dest_pos, void *stream);

/* Workspace bytes of moe_expert_ffn_q4 for T tokens. */
size_t moe_expert_ffn_workspace_size(const moe_config_t *cfg, int T);

/*
 * Grouped expert FFN on 4-bit weights (tensor cores, bf16 operands, fp32
 * accumulation): for every permuted row p of expert e,
 *   y_perm[p] = bf16( (silu(x[t] Wg_e^T) * (x[t] Wu_e^T)) Wd_e^T ),
 *   t = sorted_slot[p] / k, and the intermediate rounded to bf16;
 * and with a shared expert shared_out[t] the same FFN with its weights for
 * every token t.  x [T, H], y_perm [T k, H], shared_out [T, H] (bf16).
 * offsets [E + 1] from moe_permute.  ws: moe_expert_ffn_workspace_size
 * bytes (MOE_ERR_WORKSPACE if smaller); a wait that runs out of its budget
 * inside a kernel is recorded in ws's status word (moe_read_status).
 * Source: hipfire 0.4.3 benchmarks, "Read this before comparing columns"
 * table and the text under it (the symmetric IU4 MoE prefill route for
 * files whose experts hold symmetric int4 weights); hipEngine post, "GGUF"
 * (Q4_K).  The SwiGLU expert is this library's reading of the Qwen3 FFN.
 */
int moe_expert_ffn_q4(const moe_layer_t *L, const uint16_t *x, int T, const int32_t *sorted_slot,
                      const int32_t *offsets, uint16_t *y_perm, uint16_t *shared_out, void *ws, size_t ws_bytes,
                      void *stream);

/*
 * The two passes of moe_expert_ffn_q4, for callers that want them apart
 * (same kernels, same results):
 *   gate/up:  h[p] = bf16( silu(x[t] Wg_e^T) * (x[t] Wu_e^T) ),  h [T k (+ T), I]
 *             (fp16 instead of bf16 in the fp16-operand mode, MOE_WFMT_INT4_SYM_F16)
 *             (rows T k .. T k + T - 1 are the shared expert's, token t = p - T k)
 *   down:     y_perm[p] = bf16( h[p] Wd_e^T ), shared_out[t] = bf16( h[T k + t] Wd_s^T )
 * ws: moe_expert_ffn_workspace_size (the h buffer inside it is not used).
 */
int moe_expert_gate_up_q4(const moe_layer_t *L, const uint16_t *x, int T, const int32_t *sorted_slot,
                          const int32_t *offsets, uint16_t *h, void *ws, size_t ws_bytes, void *stream);
int moe_expert_down_q4(const moe_layer_t *L, const uint16_t *h, int T, const int32_t *offsets, uint16_t *y_perm,
                       uint16_t *shared_out, void *ws, size_t ws_bytes, void *stream);

/*
 * Weighted combine: y[t] = bf16( sum_j topk_w[t,j] y_perm[dest_pos[t k + j]]
 *                                + sigmoid(shared_gate_logit[t]) shared_out[t] )
 * summed in fp32 in j order; shared_out / shared_gate_logit may be NULL.
 * Source: the weighted sum over the chosen experts of the A3B layer
 * (hipfire 0.4.3 benchmarks, "Qwen3.6-35B-A3B prefill on the R9700"
 * table); the sigmoid gate of the shared expert is this library's reading.
 */
int moe_combine(const uint16_t *y_perm, const int32_t *dest_pos, const float *topk_w, const uint16_t *shared_out,
                const float *shared_gate_logit, int T, int H, int k, uint16_t *y, void *stream);

/*
 * Rows in a given order: out[p] = x[index[p] / k] for p < rows (x, out:
 * rows of H 16-bit values, H % 8 == 0; index values must lie in
 * [0, k * rows_of_x)).  With index = sorted_slot and k the top-k this is
 * the permuted copy of the tokens that the gate/up pass reads; with k = 1
 * it is a plain row gather (the expert-parallel layer uses it to order the
 * rows it receives by expert, and to put its results back in order).
 * Source: hipfire 0.4.3 benchmarks, "Read this before comparing columns"
 * table, row "MoE prefill route" (per-expert buffers of token rows).
 */
int moe_gather_rows(const uint16_t *x, const int32_t *index, int rows, int k, int H, uint16_t *out, void *stream);

/* --------------------------------------------------------- fused layer */

/* Workspace bytes of moe_layer_forward for up to T_max tokens. */
size_t moe_layer_workspace_size(const moe_config_t *cfg, int T_max);

/*
 * The whole layer: router logits, routing, permutation, expert FFNs and
 * combine, in that order on `stream`, with all intermediates in `ws`.
 * x [T, H] bf16 -> y [T, H] bf16.  Same kernels as the separate calls, so
 * the result is bitwise equal to running them one after another.
 */
int moe_layer_forward(const moe_layer_t *L, const uint16_t *x, int T, uint16_t *y, void *ws, size_t ws_bytes,
                      void *stream, const moe_debug_t *dbg);

/*
 * Chunked prefill: the layer over T tokens as consecutive chunks of at most
 * `chunk` tokens (the last one ragged), each a moe_layer_forward call on
 * the same stream and the same workspace, which only has to hold one chunk
 * (moe_layer_workspace_size(cfg, min(chunk, T)) bytes).  Tokens never
 * interact inside the layer, so every token's output is that of the
 * one-shot call wherever both pick the same router split (always for
 * chunk >= 4096 with E = 256, H = 2048).  The hipfire 0.4.3 benchmarks run
 * long prompts as such chunks ("Late prefill steps on mq4rs": 16000 tokens as 8192 +
 * 7808); the chunk loop is this library's.  MOE_ERR_INVALID_ARG for
 * chunk < 1; errors of a chunk stop the loop and are returned.
 */
int moe_layer_forward_chunked(const moe_layer_t *L, const uint16_t *x, int T, uint16_t *y, int chunk, void *ws,
                              size_t ws_bytes, void *stream);

/*
 * Fused decode layer: the same layer for 1 <= T <= 8 tokens as ONE
 * cooperative kernel (one CTA per SM, grid barriers between the router,
 * the gate/up and the down steps).  The pages measure decode as generated
 * tokens per second with one token per step (hipfire 0.4.3 benchmarks,
 * "Qwen3.6-35B-A3B mq4rs · decode on the R9700, 0.4.3 → 0.4.3.1", where
 * the gain comes from replaying the step's launches instead of issuing
 * them); at such sizes the separate kernels of moe_layer_forward cost more
 * in launches and pipeline fill than in memory traffic.
 *
 * Results: routing as in moe_route (on this kernel's fp32 logits); expert
 * FFNs on warp-level tensor-core MMAs with fp32 accumulation, the codes
 * entering exactly and each 32-weight chunk's scale applied to the fp32
 * result, so the weights take their exact dequantised values; h rounded to
 * bf16 once, as in moe_layer_forward.  Within the layer tolerance of the
 * oracle, but not bitwise equal to moe_layer_forward (other summation
 * order).  Independent of the number of CTAs (work is split by output rows
 * and columns with fixed K slices).  A token may list an expert more than
 * once (given ids): every place is a pair of its own.
 *
 * ws: moe_layer_decode_workspace_size(cfg, T) bytes (0 = shape or T not
 * admitted: T > 8, or x or the expert intermediates do not fit in shared
 * memory; the call then returns MOE_ERR_UNSUPPORTED).  Its first 256 bytes
 * (status word and the grid barrier's words) must be zero before the first
 * call: allocate it zeroed or call moe_read_status(ws, stream, 1, ...)
 * once.  Calls leave them valid; after MOE_ERR_TIMEOUT is recorded further
 * calls on this workspace stop at once until moe_read_status clears it.
 * dbg may export logits, gate_logit, topk_ids and topk_w, and may give
 * override_ids / override_w; its counts, offsets, sorted_slot and
 * dest_pos are not written.
 */
size_t moe_layer_decode_workspace_size(const moe_config_t *cfg, int T);
int moe_layer_decode(const moe_layer_t *L, const uint16_t *x, int T, uint16_t *y, void *ws, size_t ws_bytes,
                     void *stream, const moe_debug_t *dbg);

/*
 * Read (and, when clear != 0, reset) the device status word kept in a
 * workspace of moe_layer_forward / moe_layer_decode / moe_expert_ffn_q4 /
 * moe_permute; clearing zeroes the workspace's whole 256-byte status block.
 * Synchronises `stream`.  *status = MOE_OK or the first MOE_ERR_* code a
 * kernel recorded; *detail (optional) = where it was recorded.
 *
 * The status block (the first 256 bytes of those workspaces), as int32
 * words: [0] status, [1] detail, [16] and [18] the decode kernel's grid
 * barrier (arrival word, abort flag), [20] the wait budget in microseconds of
 * every bounded device wait of the kernels reading this workspace (0: 2 s;
 * a wait that runs out records MOE_ERR_TIMEOUT and its kernel returns with
 * its TMEM freed and its copies landed), [21] a test knob: c > 0 makes
 * CTA c - 1 of every launch reading the block drop one of its own signals
 * (moe_layer_decode: its arrival at the first grid barrier; the grouped
 * expert GEMMs: its weight copies), so that waits run out of the budget
 * (for testing the timeout path; keep it 0).  Other words are reserved and must stay zero.  The caller may
 * set words 20 and 21 with a device copy before a call; clearing resets
 * them.
 */
int moe_read_status(void *ws, void *stream, int clear, int *status, int *detail);

#ifdef __cplusplus
}
#endif

#endif /* MOEQ4_H */
