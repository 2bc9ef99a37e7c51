// C ABI of libmoeq4: argument checks, workspace layout and kernel order.
// Every step of the layer runs in the kernels of this library; the host
// code only validates, carves the caller's workspace and launches.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <cuda_runtime.h>

#include "decode.h"
#include "dequant.cuh"
#include "kernels.h"
#include "moeq4.h"

using namespace moeq4;

namespace {

thread_local char g_err[512] = "";
std::atomic<uint64_t> g_launches{0};

int fail(int code, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int ok()
{
    g_err[0] = 0;
    return MOE_OK;
}

int cuda_fail(cudaError_t e, const char *what)
{
    return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

#define REQUIRE(cond, ...)                                   \
    do {                                                     \
        if (!(cond))                                         \
            return fail(MOE_ERR_INVALID_ARG, __VA_ARGS__);   \
    } while (0)

#define REQUIRE_PTR(p)                                                                \
    do {                                                                              \
        if (!(p))                                                                     \
            return fail(MOE_ERR_INVALID_ARG, "%s: null pointer", #p);                 \
        if (!aligned16(p))                                                            \
            return fail(MOE_ERR_INVALID_ARG, "%s: not 16-byte aligned", #p);          \
    } while (0)

#define CUDA_TRY(expr, what)                     \
    do {                                         \
        cudaError_t e_ = (expr);                 \
        if (e_ != cudaSuccess)                   \
            return cuda_fail(e_, what);          \
    } while (0)

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// SMs of the current device (148 when it cannot be queried).
int device_sms()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (!n) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// CTAs of the persistent kernels: one per SM.  MOEQ4_GRID_CTAS (1 .. SM
// count) launches fewer, so that tests can give each CTA many work units
// and wrap its shared-memory rings on small problems.  Work decomposition
// (tile sizes, router K slices) never depends on it.
int num_sms()
{
    const int n = device_sms();
    const char *env = getenv("MOEQ4_GRID_CTAS");
    if (env) {
        const int g = atoi(env);
        if (g >= 1 && g < n)
            return g;
    }
    return n;
}

// Router K slices and the bytes of their partial logits (0 without a split).
int router_slices(const moe_config_t *c, int T) { return router_ksplit(T, c->E, c->H, device_sms()); }

// Bytes of the partial logits for any token count up to T (the slice count
// falls as T grows, so the largest need can come before T; it is taken at
// the ends of the 128-token steps where the slice count changes).
size_t router_part_bytes(const moe_config_t *c, int T)
{
    size_t best = 0;
    for (int t = 128; t < T + 128; t += 128) {
        const int tt = t < T ? t : T;
        const int s = router_slices(c, tt);
        const size_t b = s > 1 ? sizeof(float) * (size_t)s * tt * c->E : 0;
        best = b > best ? b : best;
    }
    return best;
}

int check_config(const moe_config_t *c)
{
    if (!c)
        return fail(MOE_ERR_INVALID_ARG, "cfg: null pointer");
    if (c->H <= 0 || c->I <= 0 || c->E <= 0 || c->k <= 0)
        return fail(MOE_ERR_INVALID_ARG, "cfg: H, I, E, k must be positive");
    if (c->wfmt != MOE_WFMT_INT4_SYM && c->wfmt != MOE_WFMT_Q4K && c->wfmt != MOE_WFMT_INT4_ASYM &&
        c->wfmt != MOE_WFMT_INT4_SYM_F16)
        return fail(MOE_ERR_UNSUPPORTED, "cfg: unknown weight format %d", c->wfmt);
    if (c->H % 128 || c->I % 128)
        return fail(MOE_ERR_UNSUPPORTED, "cfg: H (%d) and I (%d) must be multiples of 128", c->H, c->I);
    if (c->E > 1024 || c->k > 32 || c->k > c->E)
        return fail(MOE_ERR_UNSUPPORTED, "cfg: need k <= min(E, 32) and E <= 1024 (E=%d k=%d)", c->E, c->k);
    if (c->wfmt != MOE_WFMT_Q4K) {
        if (c->G < 32 || (c->G & (c->G - 1)) || c->H % c->G || c->I % c->G)
            return fail(MOE_ERR_UNSUPPORTED, "cfg: int4 group G=%d must be a power of two >= 32 dividing H and I",
                        c->G);
    } else if (c->H % 256 || c->I % 256) {
        return fail(MOE_ERR_UNSUPPORTED, "cfg: Q4K needs H and I multiples of 256");
    }
    for (int which = 0; which < 2; ++which) {
        const int nmat = which == 0 ? 2 : 1;
        const int K = which == 0 ? c->H : c->I;
        const int mb = meta_block_bytes(nmat, c->wfmt, K, c->G);
        if (mb > 32768 || gemm_smem_required(nmat, mb, c->E + 1) > 227 * 1024)
            return fail(MOE_ERR_UNSUPPORTED, "cfg: per-tile scale block of %d bytes exceeds shared memory", mb);
    }
    return MOE_OK;
}

int e_total(const moe_config_t *c) { return c->E + (c->has_shared ? 1 : 0); }

// ---------------------------------------------------------------- workspaces

struct FfnWs {
    uint16_t *h;       // [T k (+ T), I] gate/up output
    uint16_t *x_perm;  // [T k, H] token rows in permuted order (null when the caller lends a buffer)
    size_t bytes;
};

// with_xperm = false: the caller lends the permuted-row buffer (the fused
// layer lends y_perm and the shared_out buffer right after it, both dead
// until the down pass writes them).
FfnWs ffn_layout(const moe_config_t *c, int T, uint8_t *base, bool with_xperm = true)
{
    FfnWs w{};
    size_t off = 0;
    w.h = (uint16_t *)(base + off);
    off += align256(sizeof(uint16_t) * ((size_t)T * c->k + (c->has_shared ? T : 0)) * c->I);
    if (with_xperm) {
        // the routed rows, and in the fp16-operand mode the shared expert's rows after them
        w.x_perm = (uint16_t *)(base + off);
        off += align256(sizeof(uint16_t) * ((size_t)T * c->k + (c->has_shared ? T : 0)) * c->H);
    }
    w.bytes = off;
    return w;
}

struct LayerWs {
    int *status;
    float *logits, *gate_logit, *w, *router_part;
    uint16_t *router_split;
    int32_t *ids, *counts, *offsets, *sorted_slot, *dest_pos;
    void *perm_scratch;
    uint8_t *ffn;
    uint16_t *y_perm, *shared_out;
    size_t bytes;
};

LayerWs layer_layout(const moe_config_t *c, int T, uint8_t *base)
{
    LayerWs w{};
    const size_t Tk = (size_t)T * c->k;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t *p = base + off;
        off += align256(bytes);
        return p;
    };
    w.status = (int *)take(256);
    w.logits = (float *)take(sizeof(float) * (size_t)T * c->E);
    w.router_part = (float *)take(router_part_bytes(c, T));
    w.router_split = (uint16_t *)take(router_split_bytes(c->E, c->H));
    w.gate_logit = (float *)take(sizeof(float) * (size_t)T);
    w.ids = (int32_t *)take(sizeof(int32_t) * Tk);
    w.w = (float *)take(sizeof(float) * Tk);
    w.counts = (int32_t *)take(sizeof(int32_t) * c->E);
    w.offsets = (int32_t *)take(sizeof(int32_t) * (c->E + 1));
    w.sorted_slot = (int32_t *)take(sizeof(int32_t) * Tk);
    w.dest_pos = (int32_t *)take(sizeof(int32_t) * Tk);
    w.perm_scratch = take(permute_scratch_bytes(T, c->E, c->k));
    w.ffn = take(ffn_layout(c, T, nullptr, false).bytes);
    w.y_perm = (uint16_t *)take(sizeof(uint16_t) * Tk * c->H);
    w.shared_out = (uint16_t *)take(sizeof(uint16_t) * (size_t)T * c->H);
    w.bytes = off;
    return w;
}

// Workspace of the fused decode kernel: the 256-byte status block (status
// word, detail, and at byte 64 the grid barrier's arrival word, an unused
// word and the abort flag), then logits, gate logits, routing and the bf16
// gate/up outputs h.
struct DecodeWs {
    int *status;
    unsigned *bar;
    float *logits, *gate_logit, *w;
    uint16_t *h;
    int32_t *ids;
    size_t bytes;
};

DecodeWs decode_layout(const moe_config_t *c, int T, uint8_t *base)
{
    DecodeWs w{};
    const size_t Tk = (size_t)T * c->k;
    const size_t NP = Tk + (c->has_shared ? T : 0);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t *p = base + off;
        off += align256(bytes);
        return p;
    };
    w.status = (int *)take(256);
    w.bar = (unsigned *)((uint8_t *)w.status + 64);
    w.logits = (float *)take(sizeof(float) * (size_t)T * c->E);
    w.gate_logit = (float *)take(sizeof(float) * (size_t)T);
    w.ids = (int32_t *)take(sizeof(int32_t) * Tk);
    w.w = (float *)take(sizeof(float) * Tk);
    w.h = (uint16_t *)take(sizeof(uint16_t) * NP * c->I);
    w.bytes = off;
    return w;
}

constexpr size_t kMaxDynamicSmem = 227 * 1024;

// Why the decode kernel does not take (cfg, T), or null.
const char *decode_refusal(const moe_config_t *c, int T)
{
    if (T > kDecodeMaxT)
        return "the fused decode kernel takes at most 8 tokens";
    if (c->I > 1024)
        return "the fused decode kernel takes an expert intermediate of at most 1024";
    if (decode_smem_layout(T, c->k, c->H, c->I, c->has_shared, c->wfmt).bytes > kMaxDynamicSmem)
        return "x or the expert intermediates of this shape exceed shared memory";
    return nullptr;
}

int check_layer(const moe_layer_t *L)
{
    if (!L)
        return fail(MOE_ERR_INVALID_ARG, "L: null pointer");
    int rc = check_config(&L->cfg);
    if (rc)
        return rc;
    REQUIRE_PTR(L->router_w);
    if (L->router_bias)
        REQUIRE_PTR(L->router_bias);
    if (L->cfg.has_shared)
        REQUIRE_PTR(L->shared_gate);
    REQUIRE_PTR(L->gu_q);
    REQUIRE_PTR(L->gu_meta);
    REQUIRE_PTR(L->dn_q);
    REQUIRE_PTR(L->dn_meta);
    return MOE_OK;
}

// The grouped GEMMs of the expert FFN, given the permutation.
// pass: 1 = gate/up only, 2 = down only, 3 = both.  h: the intermediate
// (defaults to the one inside the FFN workspace).
int run_expert_ffn(const moe_layer_t *L, const uint16_t *x, int T, const int32_t *sorted_slot,
                   const int32_t *offsets, uint16_t *y_perm, uint16_t *shared_out, uint8_t *ffn_ws, int *status,
                   cudaStream_t st, int pass = 3, uint16_t *h = nullptr, uint16_t *x_perm = nullptr)
{
    const moe_config_t &c = L->cfg;
    const FfnWs w = ffn_layout(&c, T, ffn_ws, x_perm == nullptr);
    const int Et = e_total(&c);
    const int Tk = T * c.k;
    if (!h)
        h = w.h;
    if (!x_perm)
        x_perm = w.x_perm;
    GemmArgs a{};
    a.sorted_slot = sorted_slot;
    a.topk = c.k;
    a.Tk = Tk;
    a.offsets = offsets;
    a.E = c.E;
    a.T = T;
    a.E_total = Et;
    a.G = c.G;
    a.status = status;
    const bool f16 = c.wfmt == MOE_WFMT_INT4_SYM_F16;
    if (pass & 1) {
        // the routed experts' token rows, permuted into contiguous blocks (in
        // the fp16-operand mode as fp16, the shared expert's rows appended)
        const int shared_rows = f16 && c.has_shared ? T : 0;
        CUDA_TRY(launch_gather_rows(x, sorted_slot, Tk, c.k, c.H, x_perm, num_sms(), st, shared_rows, f16, status),
                 "gather rows");
        g_launches += 1;
        // gate/up + SwiGLU -> h [Tk + T, I]
        a.wq = (const uint8_t *)L->gu_q;
        a.wmeta = (const uint8_t *)L->gu_meta;
        a.b_src = x_perm;
        a.ldb = c.H;
        a.b_rows = Tk + shared_rows;
        a.b_src2 = c.has_shared && !f16 ? x : nullptr;
        a.b_rows2 = T;
        a.K = c.H;
        a.F = c.I / kTileRows;
        a.meta_bytes = meta_block_bytes(2, c.wfmt, c.H, c.G);
        a.out = h;
        a.out_shared = h + (size_t)Tk * c.I;
        a.ldo = c.I;
        CUDA_TRY(launch_grouped_gemm(a, 2, c.wfmt, gemm_tile_tokens(T, c.E, c.k, c.wfmt), num_sms(), st), "gate/up GEMM");
        g_launches += 1;
    }
    if (pass & 2) {
        // down -> y_perm [Tk, H], shared_out [T, H]
        a.wq = (const uint8_t *)L->dn_q;
        a.wmeta = (const uint8_t *)L->dn_meta;
        a.b_src = h;
        a.ldb = c.I;
        a.b_rows = Tk + (c.has_shared ? T : 0);
        a.b_src2 = nullptr;
        a.b_rows2 = 0;
        a.K = c.I;
        a.F = c.H / kTileRows;
        a.meta_bytes = meta_block_bytes(1, c.wfmt, c.I, c.G);
        a.out = y_perm;
        a.out_shared = shared_out;
        a.ldo = c.H;
        if (down_resident_fits(c.I, a.meta_bytes, Et))
            CUDA_TRY(launch_down_resident(a, c.wfmt, num_sms(), st), "down GEMM");
        else
            CUDA_TRY(launch_grouped_gemm(a, 1, c.wfmt, gemm_down_tile_tokens(T, c.E, c.k), num_sms(), st),
                     "down GEMM");
        g_launches += 1;
    }
    return MOE_OK;
}

}  // namespace

extern "C" {

const char *moe_last_error(void) { return g_err; }

int moe_version(void) { return 1; }

uint64_t moe_kernel_launches(void) { return g_launches.load(); }

int moe_packed_sizes(const moe_config_t *cfg, size_t *gu_q_bytes, size_t *gu_meta_bytes, size_t *dn_q_bytes,
                     size_t *dn_meta_bytes)
{
    int rc = check_config(cfg);
    if (rc)
        return rc;
    const size_t Et = (size_t)e_total(cfg);
    // codes: half a byte per weight, same count as the canonical layout
    const size_t gu_q = Et * 2 * (size_t)cfg->I * cfg->H / 2;
    const size_t dn_q = Et * (size_t)cfg->H * cfg->I / 2;
    const size_t gu_m = Et * (cfg->I / kTileRows) * (size_t)meta_block_bytes(2, cfg->wfmt, cfg->H, cfg->G);
    const size_t dn_m = Et * (cfg->H / kTileRows) * (size_t)meta_block_bytes(1, cfg->wfmt, cfg->I, cfg->G);
    if (gu_q_bytes)
        *gu_q_bytes = gu_q;
    if (gu_meta_bytes)
        *gu_meta_bytes = gu_m;
    if (dn_q_bytes)
        *dn_q_bytes = dn_q;
    if (dn_meta_bytes)
        *dn_meta_bytes = dn_m;
    return ok();
}

int moe_pack_weights(const moe_config_t *cfg, const void *gu_canon, const void *gu_scale, const void *dn_canon,
                     const void *dn_scale, void *gu_q, void *gu_meta, void *dn_q, void *dn_meta, void *stream)
{
    int rc = check_config(cfg);
    if (rc)
        return rc;
    REQUIRE(gu_canon && dn_canon, "canonical weights: null pointer");
    if (cfg->wfmt != MOE_WFMT_Q4K)
        REQUIRE(gu_scale && dn_scale, "int4 scales: null pointer");
    REQUIRE_PTR(gu_q);
    REQUIRE_PTR(gu_meta);
    REQUIRE_PTR(dn_q);
    REQUIRE_PTR(dn_meta);
    cudaStream_t st = (cudaStream_t)stream;
    CUDA_TRY(launch_pack_codes(*cfg, 0, (const uint8_t *)gu_canon, (uint8_t *)gu_q, st), "pack gate/up codes");
    CUDA_TRY(launch_pack_codes(*cfg, 1, (const uint8_t *)dn_canon, (uint8_t *)dn_q, st), "pack down codes");
    unsigned misfits = 0;
    CUDA_TRY(launch_pack_meta(*cfg, 0, (const uint8_t *)gu_canon, (const uint16_t *)gu_scale, (uint8_t *)gu_meta, st,
                              &misfits),
             "pack gate/up scales");
    CUDA_TRY(launch_pack_meta(*cfg, 1, (const uint8_t *)dn_canon, (const uint16_t *)dn_scale, (uint8_t *)dn_meta, st,
                              &misfits),
             "pack down scales");
    if (misfits)
        return fail(MOE_ERR_UNSUPPORTED,
                    "fp16-operand mode: %u scales lie outside [2^-17, 8188], where q*s is not exact in fp16", misfits);
    return ok();
}

int moe_dequant_export(const moe_config_t *cfg, const void *q, const void *meta, int which, int expert,
                       float *out_f32, uint16_t *out_bf16, void *stream)
{
    int rc = check_config(cfg);
    if (rc)
        return rc;
    REQUIRE(which == 0 || which == 1, "which must be 0 (gate/up) or 1 (down)");
    REQUIRE(expert >= 0 && expert < e_total(cfg), "expert %d out of range", expert);
    REQUIRE_PTR(q);
    REQUIRE_PTR(meta);
    REQUIRE(out_f32 || out_bf16, "no output");
    CUDA_TRY(launch_dequant_export(*cfg, which, expert, (const uint8_t *)q, (const uint8_t *)meta, out_f32, out_bf16,
                                   (cudaStream_t)stream),
             "dequant export");
    return ok();
}

size_t moe_router_workspace_size(const moe_config_t *cfg, int T)
{
    if (!cfg || T < 0 || check_config(cfg))
        return 0;
    return align256(router_part_bytes(cfg, T)) + align256(router_split_bytes(cfg->E, cfg->H)) + 256;
}

int moe_router_logits(const moe_layer_t *L, const uint16_t *x, int T, float *logits, float *gate_logit, void *ws,
                      size_t ws_bytes, void *stream)
{
    int rc = check_layer(L);
    if (rc)
        return rc;
    REQUIRE(T >= 0, "T must be >= 0");
    const size_t need = moe_router_workspace_size(&L->cfg, T);
    if (!ws || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "router workspace: need %zu bytes, got %zu", need, ws ? ws_bytes : (size_t)0);
    REQUIRE_PTR(ws);
    if (T == 0)
        return ok();
    REQUIRE_PTR(x);
    REQUIRE_PTR(logits);
    const float *g = L->cfg.has_shared && gate_logit ? L->shared_gate : nullptr;
    if (g)
        REQUIRE_PTR(gate_logit);
    cudaStream_t st = (cudaStream_t)stream;
    const int S = router_slices(&L->cfg, T);
    float *part = S > 1 ? (float *)ws : logits;
    uint16_t *wsplit = (uint16_t *)((uint8_t *)ws + align256(router_part_bytes(&L->cfg, T)));
    CUDA_TRY(launch_router_gemm(x, T, L->cfg.H, L->router_w, L->router_bias, L->cfg.E, g, part,
                                g ? gate_logit : nullptr, S, wsplit, nullptr, num_sms(), st),
             "router logits");
    g_launches += 2;
    if (S > 1) {
        CUDA_TRY(launch_router_reduce(part, S, T, L->cfg.E, L->router_bias, logits, st), "router reduce");
        g_launches += 1;
    }
    return ok();
}

int moe_route(const float *logits, int T, int E, int k, int renorm, int32_t *topk_ids, float *topk_w, void *stream)
{
    REQUIRE(T >= 0, "T must be >= 0");
    REQUIRE(E >= 1 && E <= 1024, "E must be in [1, 1024]");
    REQUIRE(k >= 1 && k <= 32 && k <= E, "k must be in [1, min(E, 32)]");
    if (T == 0)
        return ok();
    REQUIRE_PTR(logits);
    REQUIRE_PTR(topk_ids);
    REQUIRE_PTR(topk_w);
    CUDA_TRY(launch_route(logits, T, E, k, renorm, topk_ids, topk_w, (cudaStream_t)stream), "route");
    g_launches += 1;
    return ok();
}

size_t moe_permute_workspace_size(int T, int E, int k)
{
    if (T < 0 || E <= 0 || k <= 0)
        return 0;
    return 256 + permute_scratch_bytes(T, E, k);
}

int moe_permute(const int32_t *topk_ids, int T, int E, int k, int32_t *counts, int32_t *offsets, int32_t *sorted_slot,
                int32_t *dest_pos, void *ws, size_t ws_bytes, void *stream)
{
    REQUIRE(T >= 0, "T must be >= 0");
    REQUIRE(E >= 1 && E <= 1024, "E must be in [1, 1024]");
    REQUIRE(k >= 1 && k <= E, "k must be in [1, E]");
    REQUIRE((size_t)T * k < (1u << 30), "T*k too large");
    REQUIRE_PTR(counts);
    REQUIRE_PTR(offsets);
    if (!ws || ws_bytes < moe_permute_workspace_size(T, E, k))
        return fail(MOE_ERR_WORKSPACE, "permute workspace: need %zu bytes, got %zu",
                    moe_permute_workspace_size(T, E, k), ws ? ws_bytes : (size_t)0);
    REQUIRE_PTR(ws);
    if (T > 0) {
        REQUIRE_PTR(topk_ids);
        REQUIRE_PTR(sorted_slot);
        REQUIRE_PTR(dest_pos);
    }
    CUDA_TRY(launch_permute(topk_ids, T, E, k, counts, offsets, sorted_slot, dest_pos, (uint8_t *)ws + 256,
                            (int *)ws, (cudaStream_t)stream),
             "permute");
    g_launches += permute_launch_count(T, k);
    return ok();
}

int moe_permute_noalloc(const int32_t *topk_ids, int T, int E, int k, int32_t *counts, int32_t *offsets,
                        int32_t *sorted_slot, int32_t *dest_pos, void *stream)
{
    REQUIRE(T >= 0, "T must be >= 0");
    if (E < 1 || E > noalloc_max_experts())
        return fail(MOE_ERR_UNSUPPORTED,
                    "moe_permute_noalloc: E = %d is outside [1, %d], the size of its built-in scratch array", E,
                    noalloc_max_experts());
    REQUIRE(k >= 1 && k <= E, "k must be in [1, E]");
    REQUIRE((size_t)T * k < (1u << 30), "T*k too large");
    REQUIRE_PTR(counts);
    REQUIRE_PTR(offsets);
    if (T > 0) {
        REQUIRE_PTR(topk_ids);
        REQUIRE_PTR(sorted_slot);
        REQUIRE_PTR(dest_pos);
    }
    {
        // the scratch address is the current device's: the stream must belong to it
        int cur = 0, sdev = 0;
        CUDA_TRY(cudaGetDevice(&cur), "moe_permute_noalloc: cudaGetDevice");
        CUDA_TRY(cudaStreamGetDevice((cudaStream_t)stream, &sdev), "moe_permute_noalloc: cudaStreamGetDevice");
        if (sdev != cur)
            return fail(MOE_ERR_INVALID_ARG,
                        "moe_permute_noalloc: the stream belongs to device %d, the current device is %d", sdev, cur);
    }
    CUDA_TRY(launch_permute_noalloc(topk_ids, T, E, k, counts, offsets, sorted_slot, dest_pos, (cudaStream_t)stream),
             "moe_permute_noalloc");
    g_launches += (size_t)T * k > 0 ? 2 : 0;   // always the histogram and the scatter kernel
    return ok();
}

size_t moe_expert_ffn_workspace_size(const moe_config_t *cfg, int T)
{
    if (check_config(cfg) || T < 0)
        return 0;
    return 256 + ffn_layout(cfg, T, nullptr).bytes;
}

int moe_expert_ffn_q4(const moe_layer_t *L, const uint16_t *x, int T, const int32_t *sorted_slot,
                      const int32_t *offsets, uint16_t *y_perm, uint16_t *shared_out, void *ws, size_t ws_bytes,
                      void *stream)
{
    int rc = check_layer(L);
    if (rc)
        return rc;
    REQUIRE(T >= 0, "T must be >= 0");
    REQUIRE((size_t)T * (L->cfg.k + 1) < (1u << 30), "T too large");
    const size_t need = moe_expert_ffn_workspace_size(&L->cfg, T);
    if (!ws || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "expert FFN workspace: need %zu bytes, got %zu", need, ws ? ws_bytes : (size_t)0);
    REQUIRE_PTR(ws);
    if (T == 0)
        return ok();
    REQUIRE_PTR(x);
    REQUIRE_PTR(sorted_slot);
    REQUIRE_PTR(offsets);
    REQUIRE_PTR(y_perm);
    if (L->cfg.has_shared)
        REQUIRE_PTR(shared_out);
    rc = run_expert_ffn(L, x, T, sorted_slot, offsets, y_perm, shared_out, (uint8_t *)ws + 256, (int *)ws,
                        (cudaStream_t)stream);
    return rc ? rc : ok();
}

int moe_expert_gate_up_q4(const moe_layer_t *L, const uint16_t *x, int T, const int32_t *sorted_slot,
                          const int32_t *offsets, uint16_t *h, void *ws, size_t ws_bytes, void *stream)
{
    int rc = check_layer(L);
    if (rc)
        return rc;
    REQUIRE(T >= 0, "T must be >= 0");
    REQUIRE((size_t)T * (L->cfg.k + 1) < (1u << 30), "T too large");
    const size_t need = moe_expert_ffn_workspace_size(&L->cfg, T);
    if (!ws || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "expert FFN workspace: need %zu bytes, got %zu", need, ws ? ws_bytes : (size_t)0);
    REQUIRE_PTR(ws);
    if (T == 0)
        return ok();
    REQUIRE_PTR(x);
    REQUIRE_PTR(sorted_slot);
    REQUIRE_PTR(offsets);
    REQUIRE_PTR(h);
    rc = run_expert_ffn(L, x, T, sorted_slot, offsets, nullptr, nullptr, (uint8_t *)ws + 256, (int *)ws,
                        (cudaStream_t)stream, 1, h);
    return rc ? rc : ok();
}

int moe_expert_down_q4(const moe_layer_t *L, const uint16_t *h, int T, const int32_t *offsets, uint16_t *y_perm,
                       uint16_t *shared_out, void *ws, size_t ws_bytes, void *stream)
{
    int rc = check_layer(L);
    if (rc)
        return rc;
    REQUIRE(T >= 0, "T must be >= 0");
    REQUIRE((size_t)T * (L->cfg.k + 1) < (1u << 30), "T too large");
    const size_t need = moe_expert_ffn_workspace_size(&L->cfg, T);
    if (!ws || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "expert FFN workspace: need %zu bytes, got %zu", need, ws ? ws_bytes : (size_t)0);
    REQUIRE_PTR(ws);
    if (T == 0)
        return ok();
    REQUIRE_PTR(h);
    REQUIRE_PTR(offsets);
    REQUIRE_PTR(y_perm);
    if (L->cfg.has_shared)
        REQUIRE_PTR(shared_out);
    rc = run_expert_ffn(L, nullptr, T, nullptr, offsets, y_perm, shared_out, (uint8_t *)ws + 256, (int *)ws,
                        (cudaStream_t)stream, 2, const_cast<uint16_t *>(h));
    return rc ? rc : ok();
}

int moe_combine(const uint16_t *y_perm, const int32_t *dest_pos, const float *topk_w, const uint16_t *shared_out,
                const float *shared_gate_logit, int T, int H, int k, uint16_t *y, void *stream)
{
    REQUIRE(T >= 0, "T must be >= 0");
    REQUIRE(H > 0 && H % 8 == 0, "H must be a positive multiple of 8");
    REQUIRE(k >= 1 && k <= 1024, "k out of range");
    if (T == 0)
        return ok();
    REQUIRE_PTR(y_perm);
    REQUIRE_PTR(dest_pos);
    REQUIRE_PTR(topk_w);
    REQUIRE_PTR(y);
    if (shared_out)
        REQUIRE_PTR(shared_out);
    if (shared_gate_logit)
        REQUIRE_PTR(shared_gate_logit);
    CUDA_TRY(launch_combine(y_perm, dest_pos, topk_w, shared_out, shared_gate_logit, T, H, k, y, num_sms(),
                            (cudaStream_t)stream),
             "combine");
    g_launches += 1;
    return ok();
}

int moe_gather_rows(const uint16_t *x, const int32_t *index, int rows, int k, int H, uint16_t *out, void *stream)
{
    REQUIRE(rows >= 0, "rows must be >= 0");
    REQUIRE(k >= 1, "k must be >= 1");
    REQUIRE(H > 0 && H % 8 == 0, "H must be a positive multiple of 8");
    if (rows == 0)
        return ok();
    REQUIRE_PTR(x);
    REQUIRE_PTR(index);
    REQUIRE_PTR(out);
    CUDA_TRY(launch_gather_rows(x, index, rows, k, H, out, num_sms(), (cudaStream_t)stream), "gather rows");
    g_launches += 1;
    return ok();
}

size_t moe_layer_workspace_size(const moe_config_t *cfg, int T_max)
{
    if (check_config(cfg) || T_max < 0)
        return 0;
    return layer_layout(cfg, T_max, nullptr).bytes;
}

int moe_layer_forward(const moe_layer_t *L, const uint16_t *x, int T, uint16_t *y, void *ws, size_t ws_bytes,
                      void *stream, const moe_debug_t *dbg)
{
    int rc = check_layer(L);
    if (rc)
        return rc;
    const moe_config_t &c = L->cfg;
    REQUIRE(T >= 0, "T must be >= 0");
    REQUIRE((size_t)T * (c.k + 1) < (1u << 30), "T too large");
    const size_t need = moe_layer_workspace_size(&c, T);
    if (!ws || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "layer workspace: need %zu bytes, got %zu", need, ws ? ws_bytes : (size_t)0);
    REQUIRE_PTR(ws);
    if (T == 0)
        return ok();
    REQUIRE_PTR(x);
    REQUIRE_PTR(y);
    cudaStream_t st = (cudaStream_t)stream;
    const LayerWs w = layer_layout(&c, T, (uint8_t *)ws);
    const int Tk = T * c.k;
    const bool override_route = dbg && dbg->override_ids;
    if (override_route) {
        REQUIRE_PTR(dbg->override_ids);
        REQUIRE_PTR(dbg->override_w);
    }
    const float *g = c.has_shared ? L->shared_gate : nullptr;
    const int S = router_slices(&c, T);
    CUDA_TRY(launch_router_gemm(x, T, c.H, L->router_w, L->router_bias, c.E, g, S > 1 ? w.router_part : w.logits,
                                g ? w.gate_logit : nullptr, S, w.router_split, w.status, num_sms(), st),
             "router logits");
    g_launches += 2;
    const int32_t *ids = w.ids;
    const float *tw = w.w;
    if (override_route) {
        ids = dbg->override_ids;
        tw = dbg->override_w;
        if (S > 1) {
            CUDA_TRY(launch_router_reduce(w.router_part, S, T, c.E, L->router_bias, w.logits, st), "router reduce");
            g_launches += 1;
        }
    } else {
        // with split-K partials the route kernel sums them (and writes the logits)
        CUDA_TRY(launch_route(w.logits, T, c.E, c.k, c.renorm, w.ids, w.w, st, S > 1 ? w.router_part : nullptr, S,
                              L->router_bias, w.logits),
                 "route");
        g_launches += 1;
    }
    CUDA_TRY(launch_permute(ids, T, c.E, c.k, w.counts, w.offsets, w.sorted_slot, w.dest_pos, w.perm_scratch,
                            w.status, st),
             "permute");
    g_launches += permute_launch_count(T, c.k);
    rc = run_expert_ffn(L, x, T, w.sorted_slot, w.offsets, w.y_perm, c.has_shared ? w.shared_out : nullptr, w.ffn,
                        w.status, st, 3, nullptr, w.y_perm);
    if (rc)
        return rc;
    CUDA_TRY(launch_combine(w.y_perm, w.dest_pos, tw, c.has_shared ? w.shared_out : nullptr,
                            c.has_shared ? w.gate_logit : nullptr, T, c.H, c.k, y, num_sms(), st),
             "combine");
    g_launches += 1;
    if (dbg) {
        auto cp = [&](void *dst, const void *src, size_t bytes) -> cudaError_t {
            return dst ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st) : cudaSuccess;
        };
        CUDA_TRY(cp(dbg->logits, w.logits, sizeof(float) * (size_t)T * c.E), "export logits");
        if (c.has_shared)
            CUDA_TRY(cp(dbg->gate_logit, w.gate_logit, sizeof(float) * T), "export gate logit");
        CUDA_TRY(cp(dbg->topk_ids, ids, sizeof(int32_t) * Tk), "export ids");
        CUDA_TRY(cp(dbg->topk_w, tw, sizeof(float) * Tk), "export weights");
        CUDA_TRY(cp(dbg->counts, w.counts, sizeof(int32_t) * c.E), "export counts");
        CUDA_TRY(cp(dbg->offsets, w.offsets, sizeof(int32_t) * (c.E + 1)), "export offsets");
        CUDA_TRY(cp(dbg->sorted_slot, w.sorted_slot, sizeof(int32_t) * Tk), "export sorted_slot");
        CUDA_TRY(cp(dbg->dest_pos, w.dest_pos, sizeof(int32_t) * Tk), "export dest_pos");
    }
    return ok();
}

int moe_layer_forward_chunked(const moe_layer_t *L, const uint16_t *x, int T, uint16_t *y, int chunk, void *ws,
                              size_t ws_bytes, void *stream)
{
    int rc = check_layer(L);
    if (rc)
        return rc;
    REQUIRE(T >= 0, "T must be >= 0");
    REQUIRE(chunk >= 1, "chunk must be >= 1");
    const int Tc = T < chunk ? T : chunk;
    const size_t need = moe_layer_workspace_size(&L->cfg, Tc);
    if (!ws || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "layer workspace: need %zu bytes, got %zu", need, ws ? ws_bytes : (size_t)0);
    if (T == 0)
        return ok();
    REQUIRE_PTR(x);
    REQUIRE_PTR(y);
    const size_t H = (size_t)L->cfg.H;
    for (int64_t off = 0; off < T; off += chunk) {
        const int n = (int)(T - off < chunk ? T - off : chunk);
        rc = moe_layer_forward(L, x + (size_t)off * H, n, y + (size_t)off * H, ws, ws_bytes, stream, nullptr);
        if (rc)
            return rc;
    }
    return ok();
}

size_t moe_layer_decode_workspace_size(const moe_config_t *cfg, int T)
{
    if (check_config(cfg) || T < 0 || decode_refusal(cfg, T))
        return 0;
    return decode_layout(cfg, T, nullptr).bytes;
}

int moe_layer_decode(const moe_layer_t *L, const uint16_t *x, int T, uint16_t *y, void *ws, size_t ws_bytes,
                     void *stream, const moe_debug_t *dbg)
{
    int rc = check_layer(L);
    if (rc)
        return rc;
    const moe_config_t &c = L->cfg;
    REQUIRE(T >= 0, "T must be >= 0");
    if (const char *why = decode_refusal(&c, T))
        return fail(MOE_ERR_UNSUPPORTED, "moe_layer_decode: %s (T = %d)", why, T);
    const size_t need = moe_layer_decode_workspace_size(&c, T);
    if (!ws || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "decode workspace: need %zu bytes, got %zu", need, ws ? ws_bytes : (size_t)0);
    REQUIRE_PTR(ws);
    if (T == 0)
        return ok();
    REQUIRE_PTR(x);
    REQUIRE_PTR(y);
    const bool override_route = dbg && dbg->override_ids;
    if (override_route) {
        REQUIRE_PTR(dbg->override_ids);
        REQUIRE_PTR(dbg->override_w);
    }
    cudaStream_t st = (cudaStream_t)stream;
    const DecodeWs w = decode_layout(&c, T, (uint8_t *)ws);
    DecodeArgs a{};
    a.x = x;
    a.T = T;
    a.H = c.H;
    a.I = c.I;
    a.E = c.E;
    a.k = c.k;
    a.G = c.G;
    a.wfmt = c.wfmt;
    a.renorm = c.renorm;
    a.has_shared = c.has_shared ? 1 : 0;
    a.router_w = L->router_w;
    a.router_bias = L->router_bias;
    a.shared_gate = c.has_shared ? L->shared_gate : nullptr;
    a.gu_q = (const uint8_t *)L->gu_q;
    a.gu_meta = (const uint8_t *)L->gu_meta;
    a.dn_q = (const uint8_t *)L->dn_q;
    a.dn_meta = (const uint8_t *)L->dn_meta;
    a.gu_meta_bytes = meta_block_bytes(2, c.wfmt, c.H, c.G);
    a.dn_meta_bytes = meta_block_bytes(1, c.wfmt, c.I, c.G);
    a.override_ids = override_route ? dbg->override_ids : nullptr;
    a.override_w = override_route ? dbg->override_w : nullptr;
    a.logits = w.logits;
    a.gate_logit = w.gate_logit;
    a.topk_ids = w.ids;
    a.topk_w = w.w;
    a.h = w.h;
    a.y = y;
    a.status = w.status;
    a.bar = w.bar;
    CUDA_TRY(launch_decode_layer(a, num_sms(), st), "fused decode layer");
    g_launches += 1;
    if (dbg) {
        auto cp = [&](void *dst, const void *src, size_t bytes) -> cudaError_t {
            return dst ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st) : cudaSuccess;
        };
        const size_t Tk = (size_t)T * c.k;
        CUDA_TRY(cp(dbg->logits, w.logits, sizeof(float) * (size_t)T * c.E), "export logits");
        if (c.has_shared)
            CUDA_TRY(cp(dbg->gate_logit, w.gate_logit, sizeof(float) * T), "export gate logit");
        CUDA_TRY(cp(dbg->topk_ids, w.ids, sizeof(int32_t) * Tk), "export ids");
        CUDA_TRY(cp(dbg->topk_w, w.w, sizeof(float) * Tk), "export weights");
    }
    return ok();
}

int moe_read_status(void *ws, void *stream, int clear, int *status, int *detail)
{
    REQUIRE_PTR(ws);
    REQUIRE(status, "status: null pointer");
    cudaStream_t st = (cudaStream_t)stream;
    int h[2] = {0, 0};
    CUDA_TRY(cudaMemcpyAsync(h, ws, sizeof h, cudaMemcpyDeviceToHost, st), "read status");
    CUDA_TRY(cudaStreamSynchronize(st), "read status sync");
    *status = h[0];
    if (detail)
        *detail = h[1];
    if (clear) {
        // the whole status block: also the decode kernel's grid-barrier words
        CUDA_TRY(cudaMemsetAsync(ws, 0, 256, st), "clear status");
        CUDA_TRY(cudaStreamSynchronize(st), "clear status sync");
    }
    return ok();
}

}  // extern "C"
