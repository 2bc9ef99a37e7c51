"""Exact-integer GEMM pin: the down pass on integer activations and integer
codes at a power-of-two scale has an exact fp32 result (every partial sum is
a multiple of 1/8 well below 2^21), so its bf16 rounding must agree bit for
bit with the exact product rounded to nearest even.  Any misplaced row,
column, k-step or expert boundary changes bits.
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_moe_expert_warp_b200 as mq
    from quantized_moe_expert_warp_b200 import build
    build.build()
    mq.lib()
    return torch.device("cuda", 0)


def _bits_no_negzero(b):
    b = np.asarray(b, np.uint16).copy()
    b[b == 0x8000] = 0
    return b


@pytest.mark.parametrize("T,E,k,I,H,shared", [(64, 8, 2, 256, 512, True), (300, 4, 2, 256, 256, False),
                                              (1, 16, 4, 128, 256, True), (700, 3, 3, 384, 128, True)])
def test_down_gemm_exact_integers(dev, T, E, k, I, H, shared):
    import quantized_moe_expert_warp_b200 as mq
    from quantized_moe_expert_warp_b200.host import upload_layer
    G = 64
    cfg = synth.LayerConfig(name="exact", T=T, H=H, E=E, k=k, I=I, has_shared=shared,
                            wfmt=synth.WFMT_INT4_SYM, G=G, wr_std=0.05, zipf_s=0.0, seed=3)
    layer = synth.make_layer(cfg)
    rng = np.random.default_rng(T * 7 + E)
    Et = E + (1 if shared else 0)
    q = rng.integers(-8, 8, size=(Et, H, I))
    u = (q & 0xF).astype(np.uint8)
    layer["dn_nib"] = (u[..., 0::2] | (u[..., 1::2] << 4)).astype(np.uint8)
    layer["dn_scale"] = np.full((Et, H, I // G), synth.f32_to_bf16_bits(np.float32(0.125)), np.uint16)
    packed = upload_layer(layer, dev)

    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, _, _ = oracle.permute(ids, E)
    rows = T * k + (T if shared else 0)
    h = rng.integers(-2, 3, size=(rows, I)).astype(np.float32)   # exact in bf16
    h_dev = torch.from_numpy(synth.f32_to_bf16_bits(h).view(np.int16)).to(dev)
    off_dev = torch.from_numpy(offsets.astype(np.int32)).to(dev)
    y_perm = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev)
    sh = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if shared else None
    n = mq.moe_expert_ffn_workspace_size(cfg, T)
    ws = torch.zeros(n, dtype=torch.uint8, device=dev)
    mq.moe_expert_down_q4(packed, h_dev, T, off_dev, y_perm, sh, ws, n)
    status, detail = mq.moe_read_status(ws)
    assert status == 0, f"device status {status} ({detail})"

    W = q.astype(np.float64) * 0.125
    exact = np.empty((rows, H))
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        exact[a:b] = h[a:b].astype(np.float64) @ W[e].T
    if shared:
        exact[T * k:] = h[T * k:].astype(np.float64) @ W[E].T
    assert np.all(np.abs(exact) * 8 < 2 ** 21)
    want = _bits_no_negzero(synth.f32_to_bf16_bits(exact.astype(np.float32)))
    got = _bits_no_negzero(y_perm.view(torch.int16).cpu().numpy().view(np.uint16))
    assert np.array_equal(got, want[:T * k])
    if shared:
        got_s = _bits_no_negzero(sh.view(torch.int16).cpu().numpy().view(np.uint16))
        assert np.array_equal(got_s, want[T * k:])
