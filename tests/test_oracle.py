"""Pins of the CPU oracle against facts that do not come from the oracle.

Each test fixes one part of the oracle with something independent of its
code: hand-built quantised blocks with values worked out by hand, closed
forms (sigmoid values of a layer small enough to evaluate on paper),
brute force (sorting, dense evaluation of every expert on every token,
which uses neither the permutation nor the gather-combine), library
routines (numpy matmul in fp64) and invariants.
"""
import math

import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def bf16(v):
    return synth.f32_to_bf16_bits(np.asarray(v, np.float32))


def pack_nibbles(q_rows):
    """Hand packing of the canonical int4 layout, bit by bit."""
    out = []
    for row in q_rows:
        b = []
        for i in range(0, len(row), 2):
            lo = row[i] & 0xF
            hi = row[i + 1] & 0xF
            b.append(lo | (hi << 4))
        out.append(b)
    return np.array(out, np.uint8)


# --------------------------------------------------------------- dequant

def test_int4_dequant_hand_built_block():
    q = [[-8, 7, 1, -1], [0, 3, -2, 5]]
    nib = pack_nibbles(q)
    assert nib.tolist() == [[0x78, 0xF1], [0x30, 0x5E]]
    # bf16 bit patterns: 0.5, 0.25 | 0.0, 3.0
    scale = np.array([[0x3F00, 0x3E80], [0x0000, 0x4040]], np.uint16)
    w = oracle.dequant_int4sym(nib, scale, 2, 4, 2)
    assert w.tolist() == [[-4.0, 3.5, 0.25, -0.25], [0.0, 0.0, -6.0, 15.0]]


def test_int4_dequant_exact_beyond_bf16():
    # s = 1.0078125 (bf16 0x3F81); 7*s = 7.0546875 needs 11 bits: exact in fp32 only
    nib = pack_nibbles([[7, -8]])
    w = oracle.dequant_int4sym(nib, np.array([[0x3F81]], np.uint16), 1, 2, 2)
    assert w.tolist() == [[7.0546875, -8.0625]]


def test_int4_roundtrip_of_representable_weights():
    rng = np.random.default_rng(5)
    N, K, G = 6, 64, 32
    s = synth.bf16_bits_to_f32(bf16(rng.uniform(0.01, 0.05, size=(N, K // G))))
    q = rng.integers(-7, 8, size=(N, K)).astype(np.float32)
    q[:, 0] = 7          # max |w| = 7 s in each group, so the quantiser picks exactly s
    q[:, G] = -7
    w = q * np.repeat(s, G, axis=1)
    nib, sc = synth.quantize_int4_sym(w, G)
    assert np.array_equal(synth.bf16_bits_to_f32(sc), s)
    assert np.array_equal(oracle.dequant_int4sym(nib, sc, N, K, G), w)


def test_int4asym_dequant_hand_built_block():
    # unsigned codes; per group of 2: (scale, min) = (0.5, -2), (0.25, 1) | (0, 3), (2, -0.5)
    q = [[0, 15, 1, 7], [3, 0, 8, 2]]
    nib = pack_nibbles(q)
    assert nib.tolist() == [[0xF0, 0x71], [0x03, 0x28]]
    sm = np.array([[[0x3F00, 0xC000], [0x3E80, 0x3F80]],
                   [[0x0000, 0x4040], [0x4000, 0xBF00]]], np.uint16)
    w = oracle.dequant_int4asym(nib, sm, 2, 4, 2)
    assert w.tolist() == [[-2.0, 5.5, 1.25, 2.75], [3.0, 3.0, 15.5, 3.5]]


def test_int4asym_with_min_of_minus_eight_scales_is_int4sym():
    """m = -8 s and unsigned code q + 8 give the symmetric format's q s exactly
    (-8 s is exact in bf16), for the weights and for a whole layer."""
    cfg = synth.LayerConfig(name="asym_as_sym", T=11, H=64, E=5, k=2, I=32, has_shared=True,
                            wfmt=synth.WFMT_INT4_SYM, G=32, wr_std=0.3, zipf_s=0.0, seed=7)
    sym = synth.make_layer(cfg)

    def to_asym(nib, scale):
        lo, hi = nib & 0xF, nib >> 4
        u = (((lo ^ 8) | ((hi ^ 8) << 4))).astype(np.uint8)   # two's complement q -> q + 8
        s = synth.bf16_bits_to_f32(scale)
        sm = np.stack([scale, bf16(-8.0 * s)], axis=-1).astype(np.uint16)
        return u, sm

    asym = dict(sym)
    asym["cfg"] = cfg.with_(wfmt=synth.WFMT_INT4_ASYM)
    asym["gu_nib"], asym["gu_scale"] = to_asym(sym["gu_nib"], sym["gu_scale"])
    asym["dn_nib"], asym["dn_scale"] = to_asym(sym["dn_nib"], sym["dn_scale"])
    a = oracle.dequant_int4asym(asym["gu_nib"][2], asym["gu_scale"][2], 2 * cfg.I, cfg.H, cfg.G)
    b = oracle.dequant_int4sym(sym["gu_nib"][2], sym["gu_scale"][2], 2 * cfg.I, cfg.H, cfg.G)
    assert np.array_equal(a, b)
    assert np.array_equal(oracle.layer_forward(asym)["y"], oracle.layer_forward(sym)["y"])


def test_int4asym_generator_roundtrip():
    rng = np.random.default_rng(9)
    N, K, G = 8, 256, 64
    w = rng.normal(0.0, 0.02, size=(N, K)).astype(np.float32) + rng.normal(0.0, 0.01, size=(N, 1)).astype(np.float32)
    nib, sm = synth.quantize_int4_asym(w, G)
    got = oracle.dequant_int4asym(nib, sm, N, K, G)
    s = np.repeat(synth.bf16_bits_to_f32(sm[..., 0]), G, axis=1)
    m = np.repeat(synth.bf16_bits_to_f32(sm[..., 1]), G, axis=1)
    # rounding to the grid (s/2), the bf16 minimum (|m| 2^-9) and the bf16 scale at q <= 15
    bound = s / 2 + np.abs(m) * 2.0 ** -9 + 15 * s * 2.0 ** -9 + 1e-12
    assert np.all(np.abs(got - w) <= bound)
    codes = np.stack([nib & 0xF, nib >> 4], axis=-1).reshape(N, K)
    cg = codes.reshape(N, K // G, G)
    assert np.all(cg.min(axis=2) == 0) and np.all(cg.max(axis=2) >= 14)


def _q4k_block(d_bits, dmin_bits, sc, m, q):
    """Hand-built 144-byte super-block: fields placed bit by bit."""
    blk = np.zeros(144, np.uint8)
    blk[0], blk[1] = d_bits & 0xFF, d_bits >> 8
    blk[2], blk[3] = dmin_bits & 0xFF, dmin_bits >> 8
    fields = list(sc) + list(m)
    for f, v in enumerate(fields):
        for b in range(6):
            if (v >> b) & 1:
                bit = 6 * f + b
                blk[4 + bit // 8] |= 1 << (bit % 8)
    for i, v in enumerate(q):
        blk[16 + i // 2] |= (v & 0xF) << (4 * (i % 2))
    return blk


def test_q4k_dequant_hand_built_block():
    sc = [1, 2, 3, 4, 5, 6, 7, 63]
    m = [0, 1, 2, 3, 4, 5, 6, 63]
    q = [i % 16 for i in range(256)]
    blk = _q4k_block(0x3800, 0x3400, sc, m, q)     # d = 0.5, dmin = 0.25
    w = oracle.dequant_q4k(blk[None, :], 1, 256)[0]
    assert w[0] == 0.0
    assert w[1] == 0.5                 # 0.5*1*1 - 0
    assert w[32] == -0.25              # sub-block 1, q = 0: -0.25*1
    assert w[33] == 0.75               # 0.5*2*1 - 0.25
    assert w[255] == 456.75            # 0.5*63*15 - 0.25*63
    for i in range(256):
        j = i // 32
        assert w[i] == 0.5 * sc[j] * q[i] - 0.25 * m[j]


def test_q4k_dequant_edge_fields():
    # subnormal d = 2^-24, negative dmin = -0.5, sc = 0 in one sub-block
    sc = [0, 63, 1, 1, 1, 1, 1, 1]
    m = [63, 0, 1, 1, 1, 1, 1, 1]
    q = [15] * 256
    blk = _q4k_block(0x0001, 0xB800, sc, m, q)
    w = oracle.dequant_q4k(blk[None, :], 1, 256)[0]
    assert w[0] == 31.5                         # 0 - (-0.5)*63
    assert w[32] == np.float32(2.0 ** -24 * 63 * 15)
    assert w[64] == np.float32(2.0 ** -24 * 15 + 0.5)


def test_q4k_generator_roundtrip_accuracy():
    # the least-squares fit is input generation; check it produces sane codes
    rng = np.random.default_rng(3)
    w = rng.normal(0, 0.02, size=(4, 512)).astype(np.float32)
    blocks = synth.quantize_q4k(w)
    deq = oracle.dequant_q4k(blocks, 4, 512)
    rel = np.linalg.norm(deq - w) / np.linalg.norm(w)
    assert rel < 0.12


# ---------------------------------------------------------------- router

def test_router_logits_match_fp64_matmul():
    rng = np.random.default_rng(1)
    T, H, E = 9, 96, 12
    x = bf16(rng.normal(size=(T, H)))
    wr = rng.normal(0, 0.05, size=(E, H)).astype(np.float32)
    b = rng.normal(size=E).astype(np.float32)
    ref = (synth.bf16_bits_to_f32(x).astype(np.float64) @ wr.astype(np.float64).T
           + b.astype(np.float64)).astype(np.float32)
    got = oracle.router_logits(x, wr, b)
    assert np.array_equal(got, ref)


# --------------------------------------------------------------- routing

def brute_topk(row, k):
    order = sorted(range(len(row)), key=lambda e: (-float(row[e]), e))
    return order[:k]


@pytest.mark.parametrize("E,k", [(16, 2), (256, 8), (7, 7), (33, 5)])
def test_topk_matches_sort(E, k):
    rng = np.random.default_rng(E * 100 + k)
    L = rng.normal(size=(40, E)).astype(np.float32)
    L[3, :] = L[3, 0]                 # all equal
    L[5, 1::2] = L[5, 0]              # many ties
    ids, w, _ = oracle.route(L, k)
    for t in range(L.shape[0]):
        assert ids[t].tolist() == brute_topk(L[t], k)


def test_all_equal_logits():
    ids, w, w64 = oracle.route(np.zeros((1, 10), np.float32), 4)
    assert ids[0].tolist() == [0, 1, 2, 3]
    assert np.all(w64 == 0.25)


def test_signed_zero_ties_go_to_lower_id():
    L = np.array([[-0.0, 0.0, 0.0, -1.0]], np.float32)
    ids, _, _ = oracle.route(L, 2)
    assert ids[0].tolist() == [0, 1]


def test_two_logit_closed_form():
    a, b = 0.7, -1.3
    ids, w, w64 = oracle.route(np.array([[b, a]], np.float32), 2)
    assert ids[0].tolist() == [1, 0]
    d = float(np.float32(a)) - float(np.float32(b))
    assert w64[0, 0] == pytest.approx(1.0 / (1.0 + math.exp(-d)), rel=1e-15)
    assert w64[0, 1] == pytest.approx(1.0 / (1.0 + math.exp(d)), rel=1e-15)


def test_dominant_logit():
    L = np.zeros((1, 8), np.float32)
    L[0, 5] = 100.0
    ids, w, w64 = oracle.route(L, 3)
    assert ids[0].tolist() == [5, 0, 1]
    assert w64[0, 0] == pytest.approx(1.0, abs=1e-40)
    assert w64[0, 1] < 1e-40


def test_weights_invariants_and_unrenormalised_softmax():
    rng = np.random.default_rng(7)
    L = rng.normal(size=(50, 32)).astype(np.float32)
    ids, w, w64 = oracle.route(L, 6, renorm=True)
    assert np.allclose(w64.sum(1), 1.0, atol=1e-12)
    assert np.all(np.diff(w64, axis=1) <= 0)
    ids0, _, w64u = oracle.route(L, 6, renorm=False)
    assert np.array_equal(ids0, ids)
    p = np.exp(L.astype(np.float64) - L.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    assert np.allclose(w64u, np.take_along_axis(p, ids.astype(np.int64), 1), rtol=1e-12)
    # renormalising the plain probabilities gives the renormalised weights
    assert np.allclose(w64u / w64u.sum(1, keepdims=True), w64, rtol=1e-12)


def test_route_rejects_non_finite():
    L = np.zeros((1, 4), np.float32)
    L[0, 2] = np.nan
    with pytest.raises(ValueError):
        oracle.route(L, 2)


# ----------------------------------------------------------- permutation

@pytest.mark.parametrize("T,E,k", [(64, 16, 2), (5, 3, 3), (300, 256, 8), (1, 256, 8)])
def test_permutation_bruteforce_and_invariants(T, E, k):
    rng = np.random.default_rng(T + E)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, ss, dp = oracle.permute(ids, E)
    flat = ids.reshape(-1)
    ref = sorted(range(T * k), key=lambda s: (flat[s], s))
    assert ss.tolist() == ref
    assert counts.sum() == T * k
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert np.all(np.diff(offsets) == counts)
    assert np.array_equal(dp[ss], np.arange(T * k))          # bijection
    assert np.array_equal(ss[dp], np.arange(T * k))
    for e in range(E):
        seg = ss[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)
        assert np.all(flat[seg] == e)


def test_permutation_empty_experts():
    ids = np.zeros((4, 1), np.int32)
    counts, offsets, ss, dp = oracle.permute(ids, 5)
    assert counts.tolist() == [4, 0, 0, 0, 0]
    assert offsets.tolist() == [0, 4, 4, 4, 4, 4]


# ---------------------------------------------------------------- combine

def test_combine_closed_form():
    # two tokens, k = 2, H = 2; rows placed out of order by dest_pos
    Y = np.array([[1.0, 2.0], [10.0, 20.0], [100.0, 200.0], [-1.0, 0.5]])
    dest_pos = np.array([2, 0, 3, 1], np.int32)
    w = np.array([[0.75, 0.25], [0.5, 0.5]])
    S = np.array([[4.0, 8.0], [0.0, 2.0]])
    z = np.array([0.0, math.log(3.0)])          # sigmoid: 1/2 and 3/4
    y = oracle.combine(Y, dest_pos, w, S, z)
    assert y[0].tolist() == [0.75 * 100 + 0.25 * 1 + 2.0, 0.75 * 200 + 0.25 * 2 + 4.0]
    assert np.allclose(y[1], [0.5 * -1 + 0.5 * 10 + 0.0, 0.5 * 0.5 + 0.5 * 20 + 1.5], rtol=1e-15)
    assert np.array_equal(oracle.combine(Y, dest_pos, w), y - np.array([[2.0, 4.0], [0.0, 1.5]]))


# ------------------------------------------------------------- whole layer

def sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def _closed_form_layer(bias=None, k=2, renorm=True):
    """H = 2, I = 2, two routed experts + shared; every value on paper.

    x = (1, 2).  Router rows (1,0), (0,1): logits (1, 2).
    expert 0: gate rows (1,0),(0,0)  up rows (0,1),(1,0)   a=(1,0) u=(2,1)
              h = (2 sig(1), 0);  down rows (1,5),(-2,7) -> Y0 = (2s, -4s)
    expert 1: gate rows (0,.5),(0,0) up rows (2,0),(0,0)   a=(1,0) u=(2,0)
              h = (2 sig(1), 0);  down rows (3,1),(1,1)  -> Y1 = (6s, 2s)
    shared:   gate rows (1,1),(0,0)  up rows (1,0),(0,0)   a=(3,0) u=(1,0)
              h = (3 sig(3), 0);  down rows (1,0),(1,0)  -> S = (3 sig(3), 3 sig(3))
    shared gate g = (0.5, -0.25): x.g = 0, gamma = 1/2.
    """
    cfg = synth.LayerConfig(name="closed_form", T=1, H=2, E=2, k=k, I=2, has_shared=True,
                            wfmt=synth.WFMT_INT4_SYM, G=2, wr_std=0.0, zipf_s=0.0, seed=0,
                            renorm=renorm)
    gu_q = [
        [[1, 0], [0, 0], [0, 1], [1, 0]],
        [[0, 1], [0, 0], [2, 0], [0, 0]],
        [[1, 1], [0, 0], [1, 0], [0, 0]],
    ]
    gu_s = [[1.0, 1.0, 1.0, 1.0], [0.5, 1.0, 1.0, 1.0], [1.0, 1.0, 1.0, 1.0]]
    dn_q = [[[1, 5], [-2, 7]], [[3, 1], [1, 1]], [[1, 0], [1, 0]]]
    layer = {
        "cfg": cfg,
        "x": bf16([[1.0, 2.0]]),
        "router_w": np.array([[1.0, 0.0], [0.0, 1.0]], np.float32),
        "router_bias": None if bias is None else np.array(bias, np.float32),
        "shared_gate": np.array([0.5, -0.25], np.float32),
        "gu_nib": np.stack([pack_nibbles(r) for r in gu_q]),
        "gu_scale": np.stack([bf16(np.array(s)[:, None]) for s in gu_s]),
        "dn_nib": np.stack([pack_nibbles(r) for r in dn_q]),
        "dn_scale": np.stack([bf16(np.ones((2, 1))) for _ in dn_q]),
    }
    s1, s3 = sig(1.0), sig(3.0)
    Y0 = np.array([2 * s1, -4 * s1])
    Y1 = np.array([6 * s1, 2 * s1])
    S = np.array([3 * s3, 3 * s3])
    return layer, Y0, Y1, S


def test_layer_closed_form():
    layer, Y0, Y1, S = _closed_form_layer()
    r = oracle.layer_forward(layer)
    assert r["ids"].tolist() == [[1, 0]]
    want = sig(1.0) * Y1 + sig(-1.0) * Y0 + 0.5 * S
    assert np.allclose(r["y"][0], want, rtol=1e-14, atol=0)
    assert r["gate_logit"][0] == 0.0


def test_layer_closed_form_bias_tie():
    layer, Y0, Y1, S = _closed_form_layer(bias=[0.5, -0.5])   # logits (1.5, 1.5)
    r = oracle.layer_forward(layer)
    assert r["ids"].tolist() == [[0, 1]]
    assert np.allclose(r["y"][0], 0.5 * Y0 + 0.5 * Y1 + 0.5 * S, rtol=1e-14, atol=0)


def test_layer_closed_form_top1_unrenormalised():
    layer, Y0, Y1, S = _closed_form_layer(k=1, renorm=False)
    r = oracle.layer_forward(layer)
    assert r["ids"].tolist() == [[1]]
    assert np.allclose(r["y"][0], sig(1.0) * Y1 + 0.5 * S, rtol=1e-14, atol=0)


def _dequant_all(layer):
    cfg = layer["cfg"]
    H, I, Et = cfg.H, cfg.I, cfg.E_total
    gu, dn = [], []
    for e in range(Et):
        if cfg.wfmt == synth.WFMT_INT4_SYM:
            gu.append(oracle.dequant_int4sym(layer["gu_nib"][e], layer["gu_scale"][e], 2 * I, H, cfg.G))
            dn.append(oracle.dequant_int4sym(layer["dn_nib"][e], layer["dn_scale"][e], H, I, cfg.G))
        elif cfg.wfmt == synth.WFMT_INT4_ASYM:
            gu.append(oracle.dequant_int4asym(layer["gu_nib"][e], layer["gu_scale"][e], 2 * I, H, cfg.G))
            dn.append(oracle.dequant_int4asym(layer["dn_nib"][e], layer["dn_scale"][e], H, I, cfg.G))
        else:
            gu.append(oracle.dequant_q4k(layer["gu_q4k"][e], 2 * I, H))
            dn.append(oracle.dequant_q4k(layer["dn_q4k"][e], H, I))
    return np.stack(gu).astype(np.float64), np.stack(dn).astype(np.float64)


def dense_reference(layer, ids=None):
    """Every expert on every token, masked by the top-k gate (numpy, fp64).

    Shares no step with the oracle's permutation or gather-combine.  With
    ``ids`` the gate keeps those experts instead of the top k (weights still
    from the fp32 logits).
    """
    cfg = layer["cfg"]
    x = synth.bf16_bits_to_f32(layer["x"]).astype(np.float64)
    L = (x @ layer["router_w"].astype(np.float64).T)
    if layer.get("router_bias") is not None:
        L = L + layer["router_bias"].astype(np.float64)
    L32 = L.astype(np.float32)
    gate = np.zeros((cfg.T, cfg.E))
    for t in range(cfg.T):
        top = brute_topk(L32[t], cfg.k) if ids is None else np.asarray(ids[t])
        p = np.exp(L32[t].astype(np.float64) - L32[t].max())
        z = p[top].sum() if cfg.renorm else p.sum()
        gate[t, top] = p[top] / z
    gu, dn = _dequant_all(layer)
    I = cfg.I
    y = np.zeros((cfg.T, cfg.H))
    for e in range(cfg.E_total):
        a = x @ gu[e, :I].T
        u = x @ gu[e, I:].T
        h = a / (1.0 + np.exp(-a)) * u
        out = h @ dn[e].T
        if e < cfg.E:
            y += gate[:, e:e + 1] * out
        else:
            gam = 1.0 / (1.0 + np.exp(-(x @ layer["shared_gate"].astype(np.float64))))
            y += gam[:, None] * out
    return y


@pytest.mark.parametrize("variant", [
    dict(T=13, H=64, E=6, k=2, I=32, has_shared=False, G=32),
    dict(T=17, H=64, E=8, k=3, I=64, has_shared=True, G=16),
    dict(T=9, H=32, E=5, k=5, I=32, has_shared=True, G=32, renorm=False),
    dict(T=7, H=256, E=4, k=2, I=256, has_shared=True, G=256, wfmt=synth.WFMT_Q4K),
    dict(T=9, H=64, E=6, k=3, I=64, has_shared=True, G=32, wfmt=synth.WFMT_INT4_ASYM),
])
def test_layer_matches_dense_bruteforce(variant):
    v = dict(wfmt=synth.WFMT_INT4_SYM, wr_std=0.3, zipf_s=0.0, seed=11, renorm=True)
    v.update(variant)
    cfg = synth.LayerConfig(name="dense_check", **v)
    layer = synth.make_layer(cfg)
    layer["router_bias"] = np.linspace(-0.2, 0.2, cfg.E).astype(np.float32)
    got = oracle.layer_forward(layer)["y"]
    want = dense_reference(layer)
    assert np.allclose(got, want, rtol=1e-10, atol=1e-13 * np.abs(want).max())


def test_layer_sampled_rows_equal_full_rows():
    layer = synth.make_layer(synth.get_config("tiny_t64"))
    full = oracle.layer_forward(layer)["y"]
    idx = np.array([63, 0, 17, 5])
    part = oracle.layer_forward(layer, sample=idx)["y"]
    assert np.array_equal(part, full[idx])


def test_single_expert_reduces_to_dense_swiglu():
    cfg = synth.LayerConfig(name="one_expert", T=5, H=64, E=1, k=1, I=32, has_shared=False,
                            wfmt=synth.WFMT_INT4_SYM, G=32, wr_std=0.1, zipf_s=0.0, seed=3)
    layer = synth.make_layer(cfg)
    got = oracle.layer_forward(layer)
    assert np.all(got["w"] == 1.0)
    gu, dn = _dequant_all(layer)
    x = synth.bf16_bits_to_f32(layer["x"]).astype(np.float64)
    a, u = x @ gu[0, :32].T, x @ gu[0, 32:].T
    h = a * (1.0 / (1.0 + np.exp(-a))) * u
    assert np.allclose(got["y"], h @ dn[0].T, rtol=1e-12, atol=1e-15)


# ------------------------------------------- routing supplied from outside

def test_override_ids_weighed_by_oracle_closed_form():
    """Ids given without weights: the oracle weighs them from its own logits.

    Logits (1, 2).  Ids in the non-descending order (0, 1) keep the same
    softmax pair: sig(-1) for expert 0 and sig(1) for expert 1.  Top-1 on
    the lower expert: weight 1 after renormalisation, softmax over both
    (sig(-1)) without it.
    """
    layer, Y0, Y1, S = _closed_form_layer()
    r = oracle.layer_forward(layer, override_ids=np.array([[0, 1]], np.int32))
    assert np.allclose(r["w"][0], [sig(-1.0), sig(1.0)], rtol=1e-7, atol=0)
    assert np.allclose(r["y"][0], sig(-1.0) * Y0 + sig(1.0) * Y1 + 0.5 * S, rtol=1e-14, atol=0)
    layer, Y0, Y1, S = _closed_form_layer(k=1)
    r = oracle.layer_forward(layer, override_ids=np.array([[0]], np.int32))
    assert r["w"][0, 0] == 1.0
    assert np.allclose(r["y"][0], Y0 + 0.5 * S, rtol=1e-14, atol=0)
    layer, Y0, Y1, S = _closed_form_layer(k=1, renorm=False)
    r = oracle.layer_forward(layer, override_ids=np.array([[0]], np.int32))
    assert np.allclose(r["y"][0], sig(-1.0) * Y0 + 0.5 * S, rtol=1e-14, atol=0)


def test_override_ids_match_dense_bruteforce():
    """Arbitrary distinct ids per token, weighed by the oracle, against the
    dense evaluation masked by the same ids."""
    cfg = synth.LayerConfig(name="dense_override", T=11, H=64, E=7, k=3, I=32, has_shared=True,
                            wfmt=synth.WFMT_INT4_SYM, G=32, wr_std=0.3, zipf_s=0.0, seed=5)
    layer = synth.make_layer(cfg)
    rng = np.random.default_rng(4)
    ids = np.stack([rng.permutation(cfg.E)[:cfg.k] for _ in range(cfg.T)]).astype(np.int32)
    got = oracle.layer_forward(layer, override_ids=ids)
    assert np.array_equal(got["ids"], ids)
    want = dense_reference(layer, ids=ids)
    assert np.allclose(got["y"], want, rtol=1e-10, atol=1e-13 * np.abs(want).max())


def test_override_with_own_ids_is_the_plain_layer():
    layer = synth.make_layer(synth.get_config("tiny_t64"))
    plain = oracle.layer_forward(layer)
    again = oracle.layer_forward(layer, override_ids=plain["ids"])
    assert np.array_equal(again["y"], plain["y"])
    assert np.array_equal(again["w"], plain["w"])


def test_override_rejects_out_of_range_ids():
    layer = synth.make_layer(synth.get_config("tiny_t64"))
    ids = oracle.layer_forward(layer)["ids"].copy()
    ids[3, 1] = layer["cfg"].E
    with pytest.raises(ValueError):
        oracle.layer_forward(layer, override_ids=ids)
