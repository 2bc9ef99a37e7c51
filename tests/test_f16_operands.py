"""The fp16-operand mode of the int4-sym layer (MOE_WFMT_INT4_SYM_F16).

For symmetric int4 weights q * s has at most 11 significant bits, so in
fp16 every dequantised weight is exact; the tensor cores then see the
weights the oracle uses, the activations as fp16 (exact for the bf16
inputs here) and h in fp16.  These tests check: the fp16 operand of every
weight equals the oracle's exact value bit for bit; the layer matches the
oracle within the layer tolerance at small and full size; its error is
below the bf16-operand path's on the same inputs (the weight-rounding term
is gone); scales for which q * s would not be exact are refused when the
weights are packed, and activations beyond fp16's range are refused at run
time.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import check_close, compare_layer, run_layer

torch = pytest.importorskip("torch")


def small_cfg(name, **kw):
    d = dict(name=name, T=64, H=256, E=16, k=2, I=128, has_shared=False, wfmt=synth.WFMT_INT4_SYM_F16,
             G=32, wr_std=0.05, zipf_s=0.0, seed=23)
    d.update(kw)
    return synth.LayerConfig(**d)


def test_f16_mode_packs_like_int4_sym():
    """Same buffer sizes as int4-sym (the scale entry stays 16 bits)."""
    import quantized_moe_expert_warp_b200 as mq
    from quantized_moe_expert_warp_b200 import build
    build.build()
    a = synth.get_config("a3b_t512")
    b = synth.get_config("a3b_t512_f16")
    assert mq.moe_packed_sizes(a) == mq.moe_packed_sizes(b)
    # the generator draws the same weights for both
    la = synth.make_layer(a.with_T(2, "f16_cmp_a"), experts=[3])
    lb = synth.make_layer(b.with_T(2, "f16_cmp_b"), experts=[3])
    for key in ("gu_nib", "gu_scale", "dn_nib", "dn_scale"):
        assert np.array_equal(la[key], lb[key]), key


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_moe_expert_warp_b200 as mq
    from quantized_moe_expert_warp_b200 import build
    build.build()
    mq.lib()
    return torch.device("cuda", 0)


@pytest.mark.gpu
def test_f16_dequant_export_exact(dev):
    import quantized_moe_expert_warp_b200 as mq
    from quantized_moe_expert_warp_b200.host import upload_layer
    cfg = small_cfg("f16_export", H=512, I=256, E=3, G=64, has_shared=True)
    layer = synth.make_layer(cfg)
    packed = upload_layer(layer, dev)
    for e in (0, 3):
        for which, (rows, K) in enumerate([(2 * cfg.I, cfg.H), (cfg.H, cfg.I)]):
            f32 = torch.empty((rows, K), dtype=torch.float32, device=dev)
            b16 = torch.empty((rows, K), dtype=torch.int16, device=dev)
            q, meta = (packed.gu_q, packed.gu_meta) if which == 0 else (packed.dn_q, packed.dn_meta)
            mq.moe_dequant_export(cfg, q, meta, which, e, f32, b16)
            nib = layer["gu_nib"][e] if which == 0 else layer["dn_nib"][e]
            sc = layer["gu_scale"][e] if which == 0 else layer["dn_scale"][e]
            ref = oracle.dequant_int4sym(nib, sc, rows, K, cfg.G)
            assert np.array_equal(f32.cpu().numpy().view(np.uint32), ref.view(np.uint32))
            # the fp16 operand is the exact weight
            f16 = ref.astype(np.float16)
            assert np.array_equal(f16.astype(np.float32), ref)
            assert np.array_equal(b16.cpu().numpy().view(np.uint16), f16.view(np.uint16))


SMALL = [
    small_cfg("f16_tiny"),
    small_cfg("f16_ragged_shared", T=300, H=512, E=8, k=2, I=256, has_shared=True, G=64, wr_std=0.03),
    small_cfg("f16_small_tiles_shared", T=200, H=512, E=8, k=2, I=256, has_shared=True, G=128, wr_std=0.04),
    small_cfg("f16_big_groups", T=1200, H=256, E=4, k=2, I=384, G=128, wr_std=0.02, has_shared=True),
]


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_f16_layer_matches_oracle(dev, cfg):
    layer = synth.make_layer(cfg)
    got = run_layer(layer, dev)
    ref, ties, stats = compare_layer(layer, got)
    assert np.array_equal(got["sorted_slot"], ref["sorted_slot"]) or len(ties)


@pytest.mark.gpu
@pytest.mark.parametrize("name,nsample", [("a3b_t512_f16", None), ("a3b_t8192_zipf_f16", 512)])
def test_f16_full_size_layer(dev, name, nsample):
    cfg = synth.get_config(name)
    layer = synth.make_layer(cfg)
    got = run_layer(layer, dev)
    sample = None
    if nsample is not None:
        rng = np.random.default_rng(321)
        sample = np.sort(np.concatenate([[0, cfg.T - 1],
                                         rng.choice(np.arange(1, cfg.T - 1), nsample - 2, replace=False)]))
    ref, ties, stats = compare_layer(layer, got, sample=sample)
    print(f"{name}: max|err|/max|ref| {stats[0]:.2e} rel L2 {stats[1]:.2e} near-ties {len(ties)}")


@pytest.mark.gpu
def test_f16_error_below_bf16_path(dev):
    """Same weights and tokens: the fp16-operand layer is closer to the
    oracle than the bf16-operand layer (no weight rounding, h with 11
    significant bits instead of 8)."""
    out = {}
    for name in ("a3b_t512", "a3b_t512_f16"):
        cfg = synth.get_config(name).with_T(256, name + "_t256")
        layer = synth.make_layer(cfg)
        got = run_layer(layer, dev)
        _, _, stats = compare_layer(layer, got)
        out[name] = stats[1]
    print(f"rel L2: bf16 operands {out['a3b_t512']:.3e}, fp16 operands {out['a3b_t512_f16']:.3e}")
    assert out["a3b_t512_f16"] < 0.8 * out["a3b_t512"]


@pytest.mark.gpu
def test_f16_refuses_inexact_scales(dev):
    import quantized_moe_expert_warp_b200 as mq
    from quantized_moe_expert_warp_b200.host import upload_layer
    cfg = small_cfg("f16_bad_scale")
    layer = synth.make_layer(cfg)
    layer["dn_scale"] = layer["dn_scale"].copy()
    layer["dn_scale"][2, 5, 1] = synth.f32_to_bf16_bits(np.array([3e-6], np.float32))[0]   # below 2^-17
    with pytest.raises(mq.MoeError, match="not exact in fp16"):
        upload_layer(layer, dev)
    # the same weights in the bf16-operand mode are fine
    upload_layer(dict(layer, cfg=cfg.with_(wfmt=synth.WFMT_INT4_SYM)), dev)


@pytest.mark.gpu
def test_f16_refuses_activations_beyond_fp16(dev):
    import quantized_moe_expert_warp_b200 as mq
    cfg = small_cfg("f16_big_x", has_shared=True)
    layer = synth.make_layer(cfg)
    x = layer["x"].copy()
    x[7, 11] = synth.f32_to_bf16_bits(np.array([1.0e5], np.float32))[0]
    layer = dict(layer, x=x)
    with pytest.raises(AssertionError, match=f"device status {mq.MOE_ERR_UNSUPPORTED} \\(detail 40\\)"):
        run_layer(layer, dev)


@pytest.mark.gpu
def test_f16_decode_matches_oracle(dev):
    import quantized_moe_expert_warp_b200 as mq
    from quantized_moe_expert_warp_b200.host import upload_layer, x_to_device
    cfg = small_cfg("f16_decode", T=5, H=512, E=16, k=4, I=256, has_shared=True, G=64)
    layer = synth.make_layer(cfg)
    packed = upload_layer(layer, dev)
    x = x_to_device(layer["x"], dev)
    y = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)
    n = mq.moe_layer_decode_workspace_size(cfg, cfg.T)
    ws = torch.zeros(n, dtype=torch.uint8, device=dev)
    ids = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev)
    mq.moe_layer_decode(packed, x, cfg.T, y, ws, n, debug={"topk_ids": ids})
    assert mq.moe_read_status(ws) == (0, 0)
    compare_layer(layer, {"y": y.float().cpu().numpy(), "topk_ids": ids.cpu().numpy()})
