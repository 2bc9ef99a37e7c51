"""The fused decode layer (moe_layer_decode) against the CPU oracle.

Routing ids must equal the oracle's (near-ties accepted as in the other
layer tests, with the oracle re-run on the GPU's ids); outputs must meet the
layer tolerance.  The kernel splits work by output rows only, so any number
of CTAs gives the same bits; a workspace whose abort flag is raised makes
the call stop at once with MOE_ERR_TIMEOUT in the status word.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import bf16_to_f32, check_close, compare_layer, run_layer

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


def small_cfg(name, **kw):
    d = dict(name=name, T=1, H=256, E=16, k=2, I=128, has_shared=False, wfmt=synth.WFMT_INT4_SYM,
             G=32, wr_std=0.05, zipf_s=0.0, seed=31)
    d.update(kw)
    return synth.LayerConfig(**d)


def run_decode(layer, dev, packed=None, override_ids=None, override_w=None, ws=None):
    import quantized_moe_expert_warp_b200 as mq
    from quantized_moe_expert_warp_b200.host import upload_layer, x_to_device
    cfg = layer["cfg"]
    T, E, k, H = cfg.T, cfg.E, cfg.k, cfg.H
    packed = packed or upload_layer(layer, dev)
    x = x_to_device(layer["x"], dev)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    n = mq.moe_layer_decode_workspace_size(cfg, T)
    assert n > 0
    if ws is None:
        ws = torch.zeros(n, dtype=torch.uint8, device=dev)
    dbg = {"logits": torch.empty((T, E), dtype=torch.float32, device=dev),
           "gate_logit": torch.empty((T,), dtype=torch.float32, device=dev),
           "topk_ids": torch.empty((T, k), dtype=torch.int32, device=dev),
           "topk_w": torch.empty((T, k), dtype=torch.float32, device=dev)}
    if override_ids is not None:
        dbg["override_ids"] = torch.from_numpy(np.ascontiguousarray(override_ids, np.int32)).to(dev)
        dbg["override_w"] = torch.from_numpy(np.ascontiguousarray(override_w, np.float32)).to(dev)
    mq.moe_layer_decode(packed, x, T, y, ws, n, debug=dbg)
    status, detail = mq.moe_read_status(ws)
    assert status == 0, f"device status {status} (detail {detail})"
    out = {name: v.cpu().numpy() for name, v in dbg.items()}
    out["y"] = bf16_to_f32(y)
    out["y_bf16"] = y
    return out


CASES = [
    small_cfg("tiny_t1"),
    small_cfg("tiny_t5", T=5),
    # one token over many experts with a shared expert, G = 128
    small_cfg("many_experts_shared", T=1, H=512, E=64, k=8, I=128, has_shared=True, G=128),
    # eight tokens (the largest decode batch), top-8 of 64, shared expert
    small_cfg("eight_tokens", T=8, H=512, E=64, k=8, I=256, has_shared=True, G=64, wr_std=0.03),
    # Q4K super-blocks
    small_cfg("q4k_t3", T=3, H=512, E=6, k=3, I=256, has_shared=True, G=256, wfmt=synth.WFMT_Q4K),
    # asymmetric int4
    small_cfg("asym_t4", T=4, H=512, E=8, k=2, I=256, has_shared=True, G=64, wr_std=0.03,
              wfmt=synth.WFMT_INT4_ASYM),
    # top-1 without renormalisation, every token on few experts (cnt > 1 per expert)
    small_cfg("top1_norenorm_t8", T=8, H=256, E=4, k=1, I=128, renorm=False),
    # H = 384: a chunk count that is not a multiple of 8 per lane group
    small_cfg("h384", T=2, H=384, E=8, k=2, I=384, has_shared=True, G=128),
]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_decode_matches_oracle(dev, cfg):
    layer = synth.make_layer(cfg)
    got = run_decode(layer, dev)
    ref, ties, _ = compare_layer(layer, got)
    # routing weights of the (near-tie adjusted) ids: same softmax within fp32 rounding
    np.testing.assert_allclose(got["topk_w"], ref["w"], rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("name", ["a3b_decode_t1", "a3b_decode_t8"])
def test_decode_full_size(dev, name):
    cfg = synth.get_config(name)
    layer = synth.make_layer(cfg)
    got = run_decode(layer, dev)
    ref, ties, stats = compare_layer(layer, got)
    print(f"{name}: max|err|/max|ref| {stats[0]:.2e} rel L2 {stats[1]:.2e} near-ties {len(ties)}")


def test_decode_with_oracle_routing(dev):
    cfg = CASES[3]
    layer = synth.make_layer(cfg)
    ref = oracle.layer_forward(layer)
    got = run_decode(layer, dev, override_ids=ref["ids"], override_w=ref["w"])
    assert np.array_equal(got["topk_ids"], ref["ids"])
    check_close(got["y"], ref["y"], cfg.name)


def test_decode_duplicate_ids_cut_into_slots(dev):
    """A token may list an expert more than once (given ids, or NaN logits
    whose places are replaced by expert 0): every listed place is a pair of
    its own.  Expert 2 here has 14 pairs, more than the 8 columns of one
    MMA, so the kernel cuts its pairs into two slots."""
    cfg = small_cfg("duplicate_ids", T=3, H=256, E=8, k=6, I=128, has_shared=True, G=32)
    layer = synth.make_layer(cfg)
    ids = np.array([[2, 2, 2, 5, 2, 2], [2, 0, 2, 2, 7, 2], [2, 2, 1, 2, 2, 2]], np.int32)
    w = np.random.RandomState(5).uniform(0.05, 0.3, ids.shape).astype(np.float32)
    ref = oracle.layer_forward(layer, override_ids=ids, override_w=w)
    got = run_decode(layer, dev, override_ids=ids, override_w=w)
    assert np.array_equal(got["topk_ids"], ids)
    check_close(got["y"], ref["y"], cfg.name)
    # the kernel chain takes the same routing
    chain = run_layer(layer, dev, override_ids=ids, override_w=w)
    check_close(chain["y"], ref["y"], cfg.name + " (chain)")


@pytest.mark.parametrize("ctas", [1, 5])
def test_decode_independent_of_grid(dev, ctas, monkeypatch):
    from quantized_moe_expert_warp_b200.host import upload_layer
    for cfg in (CASES[3], CASES[4]):
        layer = synth.make_layer(cfg)
        packed = upload_layer(layer, dev)
        full = run_decode(layer, dev, packed=packed)
        monkeypatch.setenv("MOEQ4_GRID_CTAS", str(ctas))
        few = run_decode(layer, dev, packed=packed)
        monkeypatch.delenv("MOEQ4_GRID_CTAS")
        assert torch.equal(few["y_bf16"].view(torch.int16), full["y_bf16"].view(torch.int16))


def test_decode_repeated_calls_and_abort_flag(dev):
    """Back-to-back calls on one workspace give the same bits (the barrier
    words stay valid); a raised abort flag stops the call with
    MOE_ERR_TIMEOUT and moe_read_status clears it."""
    import quantized_moe_expert_warp_b200 as mq
    from quantized_moe_expert_warp_b200.host import upload_layer
    cfg = CASES[2]
    layer = synth.make_layer(cfg)
    packed = upload_layer(layer, dev)
    n = mq.moe_layer_decode_workspace_size(cfg, cfg.T)
    ws = torch.zeros(n, dtype=torch.uint8, device=dev)
    a = run_decode(layer, dev, packed=packed, ws=ws)["y_bf16"]
    b = run_decode(layer, dev, packed=packed, ws=ws)["y_bf16"]
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    words = ws[:256].view(torch.int32)
    assert int(words[16].item()) == 0          # barrier word back at zero (its top bit flips twice a call)
    words[18] = 1                              # abort flag, as a timed-out launch leaves it
    x = torch.zeros((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)
    y = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)
    mq.moe_layer_decode(packed, x, cfg.T, y, ws, n)
    status, detail = mq.moe_read_status(ws)    # clears the whole status block
    assert status == mq.MOE_ERR_TIMEOUT and detail == 90
    c = run_decode(layer, dev, packed=packed, ws=ws)["y_bf16"]
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))
