"""Seeded synthetic inputs for the quantized MoE expert layer.

This module only draws random numbers and writes them in the canonical
storage formats (bf16 activations, fp32 router, int4-symmetric or
Q4_K-style packed expert weights).  It holds none of the layer's
arithmetic: no dequantisation, routing, GEMM or combine.  Both the CPU
oracle (``oracle/``) and the CUDA library receive the arrays it returns.

Workload shapes follow the Qwen3.6-35B-A3B MoE layer that the hipfire
0.4.3 benchmarks page measures ("Qwen3.6-35B-A3B prefill on the R9700"
table: pp512 .. pp16384 prompts; the 8192-row prefill chunk of the
"Read this before comparing columns" table): hidden 2048, 256 routed
experts, top-8, expert intermediate 512, one shared expert.

Canonical formats (the layout both sides read):

* INT4-SYM(G): a weight matrix W [N, K] (K contiguous) is stored as
  ``nib`` uint8 [N, K/2] -- element 2i in the low nibble of byte i,
  element 2i+1 in the high nibble, two's-complement q in [-8, 7] -- and
  ``scale`` bf16 bits uint16 [N, K/G]; the weight is q * scale.
* Q4K: per 256 weights along K a 144-byte super-block: fp16 d, fp16 dmin
  (little-endian), 12 bytes holding sixteen 6-bit fields as one
  little-endian 96-bit integer (field f = bits 6f..6f+5; fields 0..7 are
  the sub-block scales sc_0..7, fields 8..15 the mins m_0..7), then 128
  bytes of unsigned 4-bit q (weight i of the block in byte i/2, low
  nibble when i is even).  Sub-block j covers weights 32j..32j+31 and
  dequantises as d*sc_j*q - dmin*m_j.

Gate and up projections of an expert are stored as one [2I, H] matrix,
gate rows first.  The down projection is [H, I].  With a shared expert
it is stored as expert index E (after the E routed experts).
"""
from __future__ import annotations

import math
import os
import hashlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, asdict
from typing import Optional

import numpy as np

__all__ = [
    "LayerConfig", "CONFIGS", "get_config", "make_layer", "f32_to_bf16_bits",
    "bf16_bits_to_f32", "quantize_int4_sym", "quantize_q4k", "f32_to_f16_bits",
]

GENERATOR_VERSION = 3

WFMT_INT4_SYM = 0
WFMT_Q4K = 1
WFMT_INT4_ASYM = 2
# the int4-sym weights computed with fp16 operands: same canonical arrays
WFMT_INT4_SYM_F16 = 3


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int            # tokens in the batch
    H: int            # hidden size
    E: int            # routed experts
    k: int            # experts per token
    I: int            # expert intermediate size
    has_shared: bool  # one always-on shared expert of intermediate I
    wfmt: int         # WFMT_INT4_SYM, WFMT_Q4K, WFMT_INT4_ASYM or WFMT_INT4_SYM_F16
    G: int            # int4-sym group size along K (256 for Q4K: super-block)
    wr_std: float     # router weight std
    zipf_s: float     # 0: no router bias; else Zipf exponent of the bias
    seed: int
    renorm: bool = True
    x_stream: int = 0  # separate activation stream (decode batches)

    @property
    def E_total(self) -> int:
        return self.E + (1 if self.has_shared else 0)

    def with_T(self, T: int, name: Optional[str] = None) -> "LayerConfig":
        d = asdict(self)
        d["T"] = T
        d["name"] = name or f"{self.name}_T{T}"
        return LayerConfig(**d)

    def with_(self, **kw) -> "LayerConfig":
        d = asdict(self)
        d.update(kw)
        return LayerConfig(**d)


def _a3b(name, T, seed, wfmt=WFMT_INT4_SYM, G=128, zipf_s=0.0, x_stream=0):
    return LayerConfig(name=name, T=T, H=2048, E=256, k=8, I=512, has_shared=True,
                       wfmt=wfmt, G=G, wr_std=0.02, zipf_s=zipf_s, seed=seed,
                       x_stream=x_stream)


CONFIGS = {
    # tiny layer the oracle finishes in well under a second
    "tiny_t64": LayerConfig(name="tiny_t64", T=64, H=256, E=16, k=2, I=128, has_shared=False,
                            wfmt=WFMT_INT4_SYM, G=32, wr_std=0.05, zipf_s=0.0, seed=0),
    # Qwen3.6-35B-A3B-shaped layer, one 512-token prefill batch
    "a3b_t512": _a3b("a3b_t512", 512, seed=1),
    # one 8192-row prefill chunk with Zipf(1.1)-skewed expert selection
    "a3b_t8192_zipf": _a3b("a3b_t8192_zipf", 8192, seed=2, zipf_s=1.1),
    # 4096 tokens, Q4_K-style super-block weights
    "a3b_t4096_q4k": _a3b("a3b_t4096_q4k", 4096, seed=3, wfmt=WFMT_Q4K, G=256),
    # asymmetric int4 (scale and minimum per group of 128), 512 tokens
    "a3b_t512_asym": _a3b("a3b_t512_asym", 512, seed=5, wfmt=WFMT_INT4_ASYM),
    # the 512-token and 8192-token layers with fp16 tensor-core operands (exact weights)
    "a3b_t512_f16": _a3b("a3b_t512_f16", 512, seed=1, wfmt=WFMT_INT4_SYM_F16),
    "a3b_t8192_zipf_f16": _a3b("a3b_t8192_zipf_f16", 8192, seed=2, zipf_s=1.1, wfmt=WFMT_INT4_SYM_F16),
    # decode-shaped batches
    "a3b_decode_t1": _a3b("a3b_decode_t1", 1, seed=4, x_stream=1),
    "a3b_decode_t8": _a3b("a3b_decode_t8", 8, seed=4, x_stream=8),
    "a3b_decode_t32": _a3b("a3b_decode_t32", 32, seed=4, x_stream=32),
}


def get_config(name: str) -> LayerConfig:
    return CONFIGS[name]


# --------------------------------------------------------------------------
# bit-level float helpers (storage conversion only)
# --------------------------------------------------------------------------

def f32_to_bf16_bits(a) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest even); returns the uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + r) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_f16_bits(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


# --------------------------------------------------------------------------
# random streams: one independent stream per (seed, tensor, index)
# --------------------------------------------------------------------------

_T_X, _T_WR, _T_BIAS, _T_PERM, _T_GATE, _T_GU, _T_DN = range(1, 8)


def _rng(seed: int, tensor: int, idx: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor, idx])))


def _normal(seed, tensor, idx, shape, std) -> np.ndarray:
    g = _rng(seed, tensor, idx)
    a = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


# --------------------------------------------------------------------------
# quantisers (input generation: they turn N(0, 0.02) draws into stored codes)
# --------------------------------------------------------------------------

def quantize_int4_sym(w: np.ndarray, G: int):
    """Symmetric int4 with one bf16 scale per G weights along K.

    scale = bf16(max|w| / 7); q = clamp(rint(w / scale), -8, 7) (q = 0 where
    the scale is 0).  Returns (nib uint8 [N, K/2], scale uint16 [N, K/G]).
    """
    N, K = w.shape
    assert K % G == 0 and K % 2 == 0
    wg = w.reshape(N, K // G, G).astype(np.float32)
    amax = np.abs(wg).max(axis=2)
    s_bits = f32_to_bf16_bits(amax / np.float32(7.0))
    s = bf16_bits_to_f32(s_bits)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(s[:, :, None] > 0, np.rint(wg / s[:, :, None]), 0.0)
    q = np.clip(q, -8, 7).astype(np.int8).reshape(N, K)
    u = (q.astype(np.uint8) & 0xF)
    nib = (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)
    return nib, s_bits


def quantize_int4_asym(w: np.ndarray, G: int):
    """Asymmetric int4 with one bf16 scale and one bf16 minimum per G weights.

    m = bf16(min w); s = bf16((max w - m) / 15); q = clamp(rint((w - m) / s),
    0, 15) (q = 0 where s = 0).  Returns (nib uint8 [N, K/2] with unsigned
    codes, element 2i in the low nibble; sm uint16 [N, K/G, 2] = (s, m)).
    """
    N, K = w.shape
    assert K % G == 0 and K % 2 == 0
    wg = w.reshape(N, K // G, G).astype(np.float32)
    m_bits = f32_to_bf16_bits(wg.min(axis=2))
    m = bf16_bits_to_f32(m_bits)
    s_bits = f32_to_bf16_bits((wg.max(axis=2) - m) / np.float32(15.0))
    s = bf16_bits_to_f32(s_bits)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(s[:, :, None] > 0, np.rint((wg - m[:, :, None]) / s[:, :, None]), 0.0)
    u = np.clip(q, 0, 15).astype(np.uint8).reshape(N, K)
    nib = (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)
    sm = np.stack([s_bits, m_bits], axis=-1).astype(np.uint16)
    return nib, sm


def _pack_6bit_fields(fields: np.ndarray) -> np.ndarray:
    """fields [..., 16] in 0..63 -> [..., 12] bytes (little-endian bitstream)."""
    f = fields.astype(np.uint64)
    lo = np.zeros(f.shape[:-1], dtype=np.uint64)
    hi = np.zeros(f.shape[:-1], dtype=np.uint64)
    for i in range(16):
        bit = 6 * i
        if bit + 6 <= 64:
            lo |= f[..., i] << np.uint64(bit)
        elif bit >= 64:
            hi |= f[..., i] << np.uint64(bit - 64)
        else:  # straddles the 64-bit boundary
            lo |= (f[..., i] << np.uint64(bit)) & np.uint64(0xFFFFFFFFFFFFFFFF)
            hi |= f[..., i] >> np.uint64(64 - bit)
    out = np.empty(f.shape[:-1] + (12,), dtype=np.uint8)
    for b in range(8):
        out[..., b] = ((lo >> np.uint64(8 * b)) & np.uint64(0xFF)).astype(np.uint8)
    for b in range(4):
        out[..., 8 + b] = ((hi >> np.uint64(8 * b)) & np.uint64(0xFF)).astype(np.uint8)
    return out


def quantize_q4k(w: np.ndarray, iters: int = 5):
    """Q4_K-style super-blocks fitted by least squares.

    Per 32-weight sub-block fit w ~ a*q - b with q in 0..15 (a few rounds of
    rint + a 2x2 least-squares solve), then quantise a_j and b_j with 6 bits
    against the fp16 super-block scales d = max a / 63 and dmin = max b / 63.
    Returns uint8 [N, K/256 * 144].
    """
    N, K = w.shape
    assert K % 256 == 0
    nb = K // 256
    x = w.reshape(N, nb, 8, 32).astype(np.float64)
    wmin = x.min(axis=3)
    wmax = x.max(axis=3)
    b = np.maximum(0.0, -wmin)
    a = (wmax + b) / 15.0
    a = np.where(a > 0, a, 1e-8)
    for _ in range(iters):
        q = np.clip(np.rint((x + b[..., None]) / a[..., None]), 0, 15)
        n = 32.0
        sq = q.sum(axis=3)
        sqq = (q * q).sum(axis=3)
        sw = x.sum(axis=3)
        sqw = (q * x).sum(axis=3)
        det = n * sqq - sq * sq
        ok = det > 1e-12
        with np.errstate(divide="ignore", invalid="ignore"):
            a_new = (n * sqw - sq * sw) / det
            b_new = (sq * sqw - sqq * sw) / det   # w ~ a*q - b  =>  b = (a*sq - sw)/n
        ok &= a_new > 0
        neg = ok & (b_new < 0)
        with np.errstate(divide="ignore", invalid="ignore"):
            a_pos = np.where(sqq > 0, sqw / sqq, a)
        a_upd = np.where(neg, a_pos, a_new)
        b_upd = np.where(neg, 0.0, b_new)
        ok2 = ok & (a_upd > 0)
        a = np.where(ok2, a_upd, a)
        b = np.where(ok2, b_upd, b)
    d = (a.max(axis=2) / 63.0).astype(np.float16)
    dmin = (b.max(axis=2) / 63.0).astype(np.float16)
    df = d.astype(np.float64)
    dmf = dmin.astype(np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        sc = np.where(df[..., None] > 0, np.clip(np.rint(a / df[..., None]), 0, 63), 0)
        m = np.where(dmf[..., None] > 0, np.clip(np.rint(b / dmf[..., None]), 0, 63), 0)
    step = df[..., None] * sc
    off = dmf[..., None] * m
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(step[..., None] > 0,
                     np.clip(np.rint((x + off[..., None]) / step[..., None]), 0, 15), 0)
    q = q.astype(np.uint8).reshape(N, nb, 256)
    qs = (q[..., 0::2] | (q[..., 1::2] << 4)).astype(np.uint8)
    fields = np.concatenate([sc, m], axis=2).astype(np.uint8)
    sm = _pack_6bit_fields(fields)
    out = np.empty((N, nb, 144), dtype=np.uint8)
    out[..., 0:2] = d.view(np.uint8).reshape(N, nb, 2)
    out[..., 2:4] = dmin.view(np.uint8).reshape(N, nb, 2)
    out[..., 4:16] = sm
    out[..., 16:144] = qs
    return out.reshape(N, nb * 144)


# --------------------------------------------------------------------------
# the layer
# --------------------------------------------------------------------------

def zipf_router_bias(cfg: LayerConfig) -> np.ndarray:
    """Per-expert logit bias that makes selection frequency follow Zipf(s).

    b_e = beta * ln p_{r(e)} with p_r proportional to r^-s over a seeded
    random permutation r of the experts and beta = sigma_L * sqrt(6) / pi,
    sigma_L = wr_std * sqrt(H) the standard deviation of an unbiased logit
    (Gumbel-max argument: adding beta*ln p to logits of spread ~beta makes
    the arg-max frequency proportional to p).
    """
    E = cfg.E
    ranks = np.arange(1, E + 1, dtype=np.float64)
    p = ranks ** (-cfg.zipf_s)
    p /= p.sum()
    perm = _rng(cfg.seed, _T_PERM).permutation(E)
    sigma_l = cfg.wr_std * math.sqrt(cfg.H)
    beta = sigma_l * math.sqrt(6.0) / math.pi
    bias = np.empty(E, dtype=np.float64)
    bias[np.arange(E)] = beta * np.log(p[perm])
    return bias.astype(np.float32)


def make_x(cfg: LayerConfig) -> np.ndarray:
    x = _normal(cfg.seed, _T_X, cfg.x_stream, (cfg.T, cfg.H), 1.0)
    return f32_to_bf16_bits(x)


def make_expert(cfg: LayerConfig, e: int):
    """Canonical quantised weights of expert e (e == E is the shared expert)."""
    H, I = cfg.H, cfg.I
    wgu = _normal(cfg.seed, _T_GU, e, (2 * I, H), 0.02)
    wdn = _normal(cfg.seed, _T_DN, e, (H, I), 0.02)
    if cfg.wfmt in (WFMT_INT4_SYM, WFMT_INT4_SYM_F16):
        return quantize_int4_sym(wgu, cfg.G) + quantize_int4_sym(wdn, cfg.G)
    if cfg.wfmt == WFMT_INT4_ASYM:
        return quantize_int4_asym(wgu, cfg.G) + quantize_int4_asym(wdn, cfg.G)
    return (quantize_q4k(wgu), quantize_q4k(wdn))


def _cache_path(cfg: LayerConfig) -> Optional[str]:
    d = os.environ.get("MOEQ4_SYNTH_CACHE")
    if not d:
        return None
    key = hashlib.sha256(repr((GENERATOR_VERSION, asdict(cfg))).encode()).hexdigest()[:16]
    return os.path.join(d, f"{cfg.name}_{key}.npz")


def make_layer(cfg: LayerConfig, experts: Optional[list] = None) -> dict:
    """All inputs of one layer call as numpy arrays (canonical formats).

    ``experts`` restricts weight generation to a subset (others are zero);
    each expert has its own random stream, so a subset equals the same
    experts of the full draw.
    """
    cache = _cache_path(cfg) if experts is None else None
    if cache and os.path.exists(cache):
        with np.load(cache) as z:
            d = {k: z[k] for k in z.files}
        d["router_bias"] = d.get("router_bias") if "router_bias" in d else None
        d["shared_gate"] = d.get("shared_gate") if "shared_gate" in d else None
        d["cfg"] = cfg
        return d
    Et = cfg.E_total
    H, I = cfg.H, cfg.I
    out = {"cfg": cfg}
    out["x"] = make_x(cfg)
    out["router_w"] = _normal(cfg.seed, _T_WR, 0, (cfg.E, H), cfg.wr_std)
    out["router_bias"] = zipf_router_bias(cfg) if cfg.zipf_s > 0 else None
    out["shared_gate"] = _normal(cfg.seed, _T_GATE, 0, (H,), 0.02) if cfg.has_shared else None
    sel = list(range(Et) if experts is None else experts)
    # experts have independent streams, so drawing them on threads is
    # deterministic; numpy releases the GIL in the bulk fills and ufuncs
    with ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1))) as ex:
        drawn = list(ex.map(lambda e: make_expert(cfg, e), sel))
    if cfg.wfmt in (WFMT_INT4_SYM, WFMT_INT4_SYM_F16):
        gu_nib = np.zeros((Et, 2 * I, H // 2), np.uint8)
        gu_sc = np.zeros((Et, 2 * I, H // cfg.G), np.uint16)
        dn_nib = np.zeros((Et, H, I // 2), np.uint8)
        dn_sc = np.zeros((Et, H, I // cfg.G), np.uint16)
        for e, (a, b, c, d) in zip(sel, drawn):
            gu_nib[e], gu_sc[e], dn_nib[e], dn_sc[e] = a, b, c, d
        out.update(gu_nib=gu_nib, gu_scale=gu_sc, dn_nib=dn_nib, dn_scale=dn_sc)
    elif cfg.wfmt == WFMT_INT4_ASYM:
        gu_nib = np.zeros((Et, 2 * I, H // 2), np.uint8)
        gu_sm = np.zeros((Et, 2 * I, H // cfg.G, 2), np.uint16)
        dn_nib = np.zeros((Et, H, I // 2), np.uint8)
        dn_sm = np.zeros((Et, H, I // cfg.G, 2), np.uint16)
        for e, (a, b, c, d) in zip(sel, drawn):
            gu_nib[e], gu_sm[e], dn_nib[e], dn_sm[e] = a, b, c, d
        out.update(gu_nib=gu_nib, gu_scale=gu_sm, dn_nib=dn_nib, dn_scale=dn_sm)
    else:
        gu = np.zeros((Et, 2 * I, H // 256 * 144), np.uint8)
        dn = np.zeros((Et, H, I // 256 * 144), np.uint8)
        for e, (a, b) in zip(sel, drawn):
            gu[e], dn[e] = a, b
        out.update(gu_q4k=gu, dn_q4k=dn)
    if cache:
        os.makedirs(os.path.dirname(cache), exist_ok=True)
        np.savez(cache + ".tmp.npz", **{k: v for k, v in out.items()
                                        if isinstance(v, np.ndarray)})
        os.replace(cache + ".tmp.npz", cache)
    return out
