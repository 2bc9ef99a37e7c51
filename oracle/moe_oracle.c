/*
 * CPU oracle for the 4-bit weight-quantized MoE expert layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library calls, links or loads
 * this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the
 * CUDA path.
 *
 * Plain, single-threaded C.  Weights are dequantised to fp32 (the formats'
 * values are exact there), every product and sum is formed in fp64, and
 * the layer output is fp64.  Routing decisions are taken on fp32 logits.
 *
 * Sources, by page:
 *  - hipfire 0.4.3 benchmarks, "Read this before comparing columns" table
 *    (row "MoE prefill route": per-expert buffers vs the symmetric IU4 MoE
 *    route) and the paragraph under it (symmetric int4 experts of the
 *    mq4rs file): the routed-expert layer whose experts hold symmetric
 *    4-bit weights.  The grouping of tokens per expert below is the
 *    "per-expert buffers" reading of that route.
 *  - hipEngine post, "GGUF" section (Q4_K_S / Q4_K_M support): the
 *    super-block 4-bit format decoded by oracle_dequant_q4k.
 *  - hipEngine post, "Implementation Notes" (KERNELS.md bullet: every
 *    kernel checked against a CPU-reference oracle): the role of this file.
 * The pages print neither the layer's equations nor a bit layout, so the
 * layer is the plainest reading of a Qwen3-family MoE FFN layer (the model
 * all pages run): softmax over router logits, top-k with lower-id ties,
 * renormalised weights, SwiGLU experts silu(x Wg^T) * (x Wu^T) then Wd,
 * a weighted sum over the k experts plus a sigmoid-gated shared expert.
 * Each such reading is marked "reading:" where it is used.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)
#define ORACLE_ENOMEM (-2)

enum { WFMT_INT4_SYM = 0, WFMT_Q4K = 1, WFMT_INT4_ASYM = 2 };

/* ---------------------------------------------------------------- scalars */

static double bf16_value(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE binary16, decoded field by field (normal, subnormal, zero). */
static double fp16_value(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);               /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);   /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* ---------------------------------------------------------- dequantisation */

/*
 * Symmetric int4 with one bf16 scale per G weights along K (the mq4rs
 * "symmetric expert" recipe; reading: scale = max|w|/7, two's-complement
 * nibbles, element 2i in the low nibble).  w[n][k] = q * s, exact in fp32.
 */
int oracle_dequant_int4sym(const uint8_t *nib, const uint16_t *scale, int64_t N, int64_t K,
                           int64_t G, float *out)
{
    if (!nib || !scale || !out || N < 0 || K <= 0 || G <= 0 || K % G || K % 2)
        return ORACLE_EINVAL;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = nib[n * (K / 2) + k / 2];
            int u = (k & 1) ? (byte >> 4) : (byte & 0xF);
            int q = u >= 8 ? u - 16 : u;
            double s = bf16_value(scale[n * (K / G) + k / G]);
            out[n * K + k] = (float)(q * s);
        }
    }
    return ORACLE_OK;
}

/*
 * Asymmetric int4 (the mq4r file's experts, hipfire 0.4.3 benchmarks,
 * "Read this before comparing columns"; reading: one bf16 scale s and one
 * bf16 minimum m per G weights along K, unsigned 4-bit q, as in the GGUF
 * Q4_1 family).  sm holds the pairs (s, m) per group: [N, K/G, 2].
 * w[n][k] = q * s + m, formed exactly in fp64 and rounded once to fp32.
 */
int oracle_dequant_int4asym(const uint8_t *nib, const uint16_t *sm, int64_t N, int64_t K, int64_t G,
                            float *out)
{
    if (!nib || !sm || !out || N < 0 || K <= 0 || G <= 0 || K % G || K % 2)
        return ORACLE_EINVAL;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = nib[n * (K / 2) + k / 2];
            int q = (k & 1) ? (byte >> 4) : (byte & 0xF);
            const uint16_t *p = sm + (n * (K / G) + k / G) * 2;
            out[n * K + k] = (float)(q * bf16_value(p[0]) + bf16_value(p[1]));
        }
    }
    return ORACLE_OK;
}

/* six-bit field f (0..15) of the 12-byte little-endian bit stream */
static int field6(const uint8_t *sm, int f)
{
    int v = 0;
    for (int b = 0; b < 6; ++b) {
        int bit = 6 * f + b;
        v |= ((sm[bit / 8] >> (bit % 8)) & 1) << b;
    }
    return v;
}

/*
 * Q4_K-style super-block (GGUF Q4_K family named in the hipEngine post):
 * 256 weights, 8 sub-blocks of 32; w = d*sc_j*q - dmin*m_j.  Every product
 * is exact in fp64 and the difference is rounded once to fp32.
 */
int oracle_dequant_q4k(const uint8_t *blocks, int64_t N, int64_t K, float *out)
{
    if (!blocks || !out || N < 0 || K <= 0 || K % 256)
        return ORACLE_EINVAL;
    const int64_t nb = K / 256;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < nb; ++b) {
            const uint8_t *blk = blocks + (n * nb + b) * 144;
            double d = fp16_value((uint16_t)(blk[0] | (blk[1] << 8)));
            double dmin = fp16_value((uint16_t)(blk[2] | (blk[3] << 8)));
            const uint8_t *sm = blk + 4;
            const uint8_t *qs = blk + 16;
            for (int i = 0; i < 256; ++i) {
                int j = i / 32;
                int sc = field6(sm, j);
                int m = field6(sm, 8 + j);
                int q = (i & 1) ? (qs[i / 2] >> 4) : (qs[i / 2] & 0xF);
                out[n * K + b * 256 + i] = (float)(d * sc * q - dmin * m);
            }
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ router */

/* logits[t][e] = fp32( sum_h x[t][h] * Wr[e][h] + bias[e] ), summed in fp64 */
int oracle_router_logits(const uint16_t *x, int64_t T, int64_t H, const float *wr,
                         const float *bias, int64_t E, float *logits)
{
    if (!x || !wr || !logits || T < 0 || H <= 0 || E <= 0)
        return ORACLE_EINVAL;
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t h = 0; h < H; ++h)
                acc += bf16_value(x[t * H + h]) * (double)wr[e * H + h];
            if (bias)
                acc += (double)bias[e];
            logits[t * E + e] = (float)acc;
        }
    }
    return ORACLE_OK;
}

/*
 * Top-k of one token's fp32 logits: larger logit first, equal logits by
 * lower expert id (reading; the pages give no tie rule).  Output order is
 * descending.  Weights: softmax restricted to the k chosen experts
 * (renorm = 1: equal to softmax over all E followed by renormalisation of
 * the chosen k) or the plain softmax probability over all E (renorm = 0).
 */
/* Weights of k chosen experts from the token's fp32 logits (the chosen ids
 * in any order, the first taken as the reference for exp): softmax over the
 * k chosen logits (renorm = 1) or over all E (renorm = 0). */
static void topk_weights(const float *L, int64_t E, int64_t k, int renorm, const int32_t *ids, double *w)
{
    double top = (double)L[ids[0]];
    double z = 0.0;
    if (renorm) {
        for (int64_t j = 0; j < k; ++j)
            z += exp((double)L[ids[j]] - top);
    } else {
        for (int64_t e = 0; e < E; ++e)
            z += exp((double)L[e] - top);
    }
    for (int64_t j = 0; j < k; ++j)
        w[j] = exp((double)L[ids[j]] - top) / z;
}

static void route_one(const float *L, int64_t E, int64_t k, int renorm, int32_t *ids, double *w)
{
    for (int64_t j = 0; j < k; ++j) {
        int64_t best = -1;
        for (int64_t e = 0; e < E; ++e) {
            int taken = 0;
            for (int64_t i = 0; i < j; ++i)
                if (ids[i] == e)
                    taken = 1;
            if (taken)
                continue;
            if (best < 0 || L[e] > L[best])
                best = e;        /* strict '>' keeps the lower id on ties */
        }
        ids[j] = (int32_t)best;
    }
    topk_weights(L, E, k, renorm, ids, w);
}

int oracle_route(const float *logits, int64_t T, int64_t E, int64_t k, int renorm, int32_t *ids,
                 float *w32, double *w64)
{
    if (!logits || !ids || T < 0 || E <= 0 || k <= 0 || k > E)
        return ORACLE_EINVAL;
    double *w = (double *)malloc(sizeof(double) * (size_t)k);
    if (!w)
        return ORACLE_ENOMEM;
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t e = 0; e < E; ++e)
            if (!isfinite(logits[t * E + e])) {
                free(w);
                return ORACLE_EINVAL;
            }
        route_one(logits + t * E, E, k, renorm, ids + t * k, w);
        for (int64_t j = 0; j < k; ++j) {
            if (w32)
                w32[t * k + j] = (float)w[j];
            if (w64)
                w64[t * k + j] = w[j];
        }
    }
    free(w);
    return ORACLE_OK;
}

/* ------------------------------------------------------------- permutation */

/*
 * Counting sort of the T*k slots (slot = t*k + j) by expert: counts,
 * exclusive offsets (offsets[E] = T*k), and inside an expert the slots in
 * increasing slot order ("per-expert buffers", filled in token order).
 * sorted_slot[p] = slot, dest_pos[slot] = p.
 */
int oracle_permute(const int32_t *ids, int64_t T, int64_t E, int64_t k, int32_t *counts,
                   int32_t *offsets, int32_t *sorted_slot, int32_t *dest_pos)
{
    if (!ids || !counts || !offsets || !sorted_slot || !dest_pos || T < 0 || E <= 0 || k <= 0)
        return ORACLE_EINVAL;
    const int64_t S = T * k;
    for (int64_t e = 0; e < E; ++e)
        counts[e] = 0;
    for (int64_t s = 0; s < S; ++s) {
        if (ids[s] < 0 || ids[s] >= E)
            return ORACLE_EINVAL;
        counts[ids[s]]++;
    }
    offsets[0] = 0;
    for (int64_t e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];
    int32_t *fill = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    if (!fill)
        return ORACLE_ENOMEM;
    for (int64_t s = 0; s < S; ++s) {
        int32_t e = ids[s];
        int32_t p = offsets[e] + fill[e]++;
        sorted_slot[p] = (int32_t)s;
        dest_pos[s] = p;
    }
    free(fill);
    return ORACLE_OK;
}

/* -------------------------------------------------------------- combine */

/*
 * y[t] = sum_{j<k} w[t][j] * Y[dest_pos[t k + j]] + sigmoid(z[t]) * S[t]
 * for given expert outputs Y [T k, H] and shared outputs S [T, H] (S and z
 * may be NULL: no shared term).  Sums in fp64, j in order.
 */
int oracle_combine(const double *Y, const int32_t *dest_pos, const double *w, const double *S,
                   const double *z, int64_t T, int64_t H, int64_t k, double *y)
{
    if (!Y || !dest_pos || !w || !y || T < 0 || H <= 0 || k <= 0)
        return ORACLE_EINVAL;
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t c = 0; c < H; ++c) {
            double acc = 0.0;
            for (int64_t j = 0; j < k; ++j) {
                int32_t p = dest_pos[t * k + j];
                if (p < 0 || p >= T * k)
                    return ORACLE_EINVAL;
                acc += w[t * k + j] * Y[(int64_t)p * H + c];
            }
            if (S && z)
                acc += 1.0 / (1.0 + exp(-z[t])) * S[t * H + c];
            y[t * H + c] = acc;
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------ expert FFN */

static double silu(double a) { return a / (1.0 + exp(-a)); }

/*
 * One SwiGLU expert on one token (reading: gate rows first in the [2I, H]
 * gate/up matrix):  a = x Wg^T, u = x Wu^T, h = silu(a) * u, out = h Wd^T.
 */
static void expert_ffn(const double *x, int64_t H, int64_t I, const float *wgu, const float *wdn,
                       double *h, double *out)
{
    for (int64_t i = 0; i < I; ++i) {
        double a = 0.0, u = 0.0;
        for (int64_t c = 0; c < H; ++c) {
            a += x[c] * (double)wgu[i * H + c];
            u += x[c] * (double)wgu[(I + i) * H + c];
        }
        h[i] = silu(a) * u;
    }
    for (int64_t o = 0; o < H; ++o) {
        double acc = 0.0;
        for (int64_t i = 0; i < I; ++i)
            acc += h[i] * (double)wdn[o * I + i];
        out[o] = acc;
    }
}

typedef struct {
    /* shapes */
    int64_t T, H, E, k, I;
    int32_t has_shared, wfmt, G, renorm;
    /* inputs (host) */
    const uint16_t *x;           /* [T, H] bf16 bits */
    const float *router_w;       /* [E, H] */
    const float *router_bias;    /* [E] or NULL */
    const float *shared_gate;    /* [H] (has_shared) */
    const uint8_t *gu_q;         /* int4: nib [Et, 2I, H/2]; Q4K: [Et, 2I, H/256*144] */
    const uint16_t *gu_scale;    /* int4-sym: [Et, 2I, H/G]; int4-asym: [Et, 2I, H/G, 2]; Q4K: NULL */
    const uint8_t *dn_q;         /* int4: nib [Et, H, I/2]; Q4K: [Et, H, I/256*144] */
    const uint16_t *dn_scale;    /* int4-sym: [Et, H, I/G]; int4-asym: [Et, H, I/G, 2]; Q4K: NULL */
    const int32_t *override_ids; /* optional [T, k]: routing to use instead of the oracle's */
    const float *override_w;     /* optional [T, k] (with override_ids); NULL: the oracle weighs
                                    the given ids itself from its own logits */
    const int32_t *sample;       /* tokens whose output rows are computed; NULL = all */
    int64_t n_sample;
    /* outputs */
    double *y;                   /* [n_sample (or T), H] */
    float *logits;               /* optional [T, E] */
    double *gate_logit;          /* optional [T] */
    int32_t *ids;                /* optional [T, k] */
    float *w;                    /* optional [T, k] */
    int32_t *counts;             /* optional [E] */
    int32_t *offsets;            /* optional [E + 1] */
    int32_t *sorted_slot;        /* optional [T k] */
    int32_t *dest_pos;           /* optional [T k] */
} oracle_layer_args;

static int dequant_expert(const oracle_layer_args *A, int64_t e, float *wgu, float *wdn)
{
    const int64_t H = A->H, I = A->I;
    if (A->wfmt == WFMT_INT4_SYM) {
        int rc = oracle_dequant_int4sym(A->gu_q + e * (2 * I) * (H / 2),
                                        A->gu_scale + e * (2 * I) * (H / A->G), 2 * I, H, A->G, wgu);
        if (rc)
            return rc;
        return oracle_dequant_int4sym(A->dn_q + e * H * (I / 2), A->dn_scale + e * H * (I / A->G), H,
                                      I, A->G, wdn);
    }
    if (A->wfmt == WFMT_INT4_ASYM) {
        int rc = oracle_dequant_int4asym(A->gu_q + e * (2 * I) * (H / 2),
                                         A->gu_scale + e * (2 * I) * (H / A->G) * 2, 2 * I, H, A->G, wgu);
        if (rc)
            return rc;
        return oracle_dequant_int4asym(A->dn_q + e * H * (I / 2), A->dn_scale + e * H * (I / A->G) * 2, H,
                                       I, A->G, wdn);
    }
    if (A->wfmt == WFMT_Q4K) {
        int rc = oracle_dequant_q4k(A->gu_q + e * (2 * I) * (H / 256 * 144), 2 * I, H, wgu);
        if (rc)
            return rc;
        return oracle_dequant_q4k(A->dn_q + e * H * (I / 256 * 144), H, I, wdn);
    }
    return ORACLE_EINVAL;
}

/*
 * The whole layer, step by step in the order of the hot path: router
 * logits, top-k routing, permutation by expert, per-expert SwiGLU FFN over
 * the expert's rows, then per token the weighted sum over its k experts
 * plus the shared expert scaled by sigmoid(x . g) (reading: the shared
 * expert's gate is a sigmoid of one dot product with a [H] vector, no
 * bias).  Only the rows of the sampled tokens go through the FFN.
 */
int oracle_layer_forward(const oracle_layer_args *A)
{
    if (!A || !A->x || !A->router_w || !A->gu_q || !A->dn_q || !A->y)
        return ORACLE_EINVAL;
    const int64_t T = A->T, H = A->H, E = A->E, k = A->k, I = A->I;
    if (T < 0 || H <= 0 || E <= 0 || k <= 0 || k > E || I <= 0)
        return ORACLE_EINVAL;
    if ((A->wfmt == WFMT_INT4_SYM || A->wfmt == WFMT_INT4_ASYM) && (!A->gu_scale || !A->dn_scale || A->G <= 0))
        return ORACLE_EINVAL;
    if (A->has_shared && !A->shared_gate)
        return ORACLE_EINVAL;
    const int64_t S = T * k;
    const int64_t ns = A->sample ? A->n_sample : T;
    int rc = ORACLE_ENOMEM;

    float *logits = (float *)malloc(sizeof(float) * (size_t)(T * E + 1));
    int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * (size_t)(S + 1));
    double *w = (double *)malloc(sizeof(double) * (size_t)(S + 1));
    int32_t *counts = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    int32_t *offsets = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t *sorted_slot = (int32_t *)malloc(sizeof(int32_t) * (size_t)(S + 1));
    int32_t *dest_pos = (int32_t *)malloc(sizeof(int32_t) * (size_t)(S + 1));
    int64_t *row_of_tok = (int64_t *)malloc(sizeof(int64_t) * (size_t)(T + 1)); /* token -> sample row */
    int64_t *yrow = (int64_t *)malloc(sizeof(int64_t) * (size_t)(S + 1));      /* perm row -> Y row */
    float *wgu = (float *)malloc(sizeof(float) * (size_t)(2 * I * H));
    float *wdn = (float *)malloc(sizeof(float) * (size_t)(H * I));
    double *xr = (double *)malloc(sizeof(double) * (size_t)H);
    double *hbuf = (double *)malloc(sizeof(double) * (size_t)I);
    double *Y = NULL, *Sh = NULL;
    if (!logits || !ids || !w || !counts || !offsets || !sorted_slot || !dest_pos || !row_of_tok ||
        !yrow || !wgu || !wdn || !xr || !hbuf)
        goto done;

    /* 1. router logits (fp64 sums, fp32 result) */
    rc = oracle_router_logits(A->x, T, H, A->router_w, A->router_bias, E, logits);
    if (rc)
        goto done;
    /* 2. routing */
    if (A->override_ids) {
        for (int64_t s = 0; s < S; ++s) {
            ids[s] = A->override_ids[s];
            if (ids[s] < 0 || ids[s] >= E) {
                rc = ORACLE_EINVAL;
                goto done;
            }
            if (A->override_w)
                w[s] = (double)A->override_w[s];
        }
        if (!A->override_w)
            for (int64_t t = 0; t < T; ++t)
                topk_weights(logits + t * E, E, k, A->renorm, ids + t * k, w + t * k);
    } else {
        rc = oracle_route(logits, T, E, k, A->renorm, ids, NULL, w);
        if (rc)
            goto done;
    }
    /* 3. permutation */
    rc = oracle_permute(ids, T, E, k, counts, offsets, sorted_slot, dest_pos);
    if (rc)
        goto done;

    /* which tokens are wanted, and a Y row for every permuted row of them */
    for (int64_t t = 0; t < T; ++t)
        row_of_tok[t] = -1;
    for (int64_t i = 0; i < ns; ++i) {
        int64_t t = A->sample ? A->sample[i] : i;
        if (t < 0 || t >= T) {
            rc = ORACLE_EINVAL;
            goto done;
        }
        row_of_tok[t] = i;
    }
    int64_t nY = 0;
    for (int64_t p = 0; p < S; ++p)
        yrow[p] = row_of_tok[sorted_slot[p] / k] >= 0 ? nY++ : -1;
    Y = (double *)malloc(sizeof(double) * (size_t)((nY + 1) * H));
    if (A->has_shared)
        Sh = (double *)malloc(sizeof(double) * (size_t)((ns + 1) * H));
    if (!Y || (A->has_shared && !Sh)) {
        rc = ORACLE_ENOMEM;
        goto done;
    }

    /* 4-5. routed experts, each over its contiguous rows of the permutation */
    for (int64_t e = 0; e < E; ++e) {
        int any = 0;
        for (int64_t p = offsets[e]; p < offsets[e + 1]; ++p)
            any |= yrow[p] >= 0;
        if (!any)
            continue;
        rc = dequant_expert(A, e, wgu, wdn);
        if (rc)
            goto done;
        for (int64_t p = offsets[e]; p < offsets[e + 1]; ++p) {
            if (yrow[p] < 0)
                continue;
            int64_t t = sorted_slot[p] / k;
            for (int64_t c = 0; c < H; ++c)
                xr[c] = bf16_value(A->x[t * H + c]);
            expert_ffn(xr, H, I, wgu, wdn, hbuf, Y + yrow[p] * H);
        }
    }
    /* shared expert: every wanted token */
    if (A->has_shared) {
        rc = dequant_expert(A, E, wgu, wdn);
        if (rc)
            goto done;
        for (int64_t i = 0; i < ns; ++i) {
            int64_t t = A->sample ? A->sample[i] : i;
            for (int64_t c = 0; c < H; ++c)
                xr[c] = bf16_value(A->x[t * H + c]);
            expert_ffn(xr, H, I, wgu, wdn, hbuf, Sh + i * H);
        }
    }

    /* 6. combine: y[t] = sum_j w[t][j] Y[dest_pos[t k + j]] + sigmoid(x[t].g) S[t] */
    for (int64_t i = 0; i < ns; ++i) {
        int64_t t = A->sample ? A->sample[i] : i;
        double *yo = A->y + i * H;
        for (int64_t c = 0; c < H; ++c)
            yo[c] = 0.0;
        for (int64_t j = 0; j < k; ++j) {
            const double *Yr = Y + yrow[dest_pos[t * k + j]] * H;
            for (int64_t c = 0; c < H; ++c)
                yo[c] += w[t * k + j] * Yr[c];
        }
        if (A->has_shared) {
            double z = 0.0;
            for (int64_t c = 0; c < H; ++c)
                z += bf16_value(A->x[t * H + c]) * (double)A->shared_gate[c];
            double gamma = 1.0 / (1.0 + exp(-z));
            for (int64_t c = 0; c < H; ++c)
                yo[c] += gamma * Sh[i * H + c];
        }
    }

    /* optional exports */
    if (A->gate_logit && A->has_shared) {
        for (int64_t t = 0; t < T; ++t) {
            double z = 0.0;
            for (int64_t c = 0; c < H; ++c)
                z += bf16_value(A->x[t * H + c]) * (double)A->shared_gate[c];
            A->gate_logit[t] = z;
        }
    }
    if (A->logits)
        memcpy(A->logits, logits, sizeof(float) * (size_t)(T * E));
    for (int64_t s = 0; s < S; ++s) {
        if (A->ids)
            A->ids[s] = ids[s];
        if (A->w)
            A->w[s] = (float)w[s];
        if (A->sorted_slot)
            A->sorted_slot[s] = sorted_slot[s];
        if (A->dest_pos)
            A->dest_pos[s] = dest_pos[s];
    }
    if (A->counts)
        memcpy(A->counts, counts, sizeof(int32_t) * (size_t)E);
    if (A->offsets)
        memcpy(A->offsets, offsets, sizeof(int32_t) * (size_t)(E + 1));
    rc = ORACLE_OK;
done:
    free(logits);
    free(ids);
    free(w);
    free(counts);
    free(offsets);
    free(sorted_slot);
    free(dest_pos);
    free(row_of_tok);
    free(yrow);
    free(wgu);
    free(wdn);
    free(xr);
    free(hbuf);
    free(Y);
    free(Sh);
    return rc;
}
