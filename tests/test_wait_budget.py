"""The bounded device waits run out cleanly.

Every wait in the kernels gives up after the workspace's wait budget (word
20 of its 256-byte status block, in microseconds; 0 means 2 s), records
MOE_ERR_TIMEOUT in the status word and lets the kernel return, with TMEM
freed and its own copies landed.  These tests make waits run out on
purpose without any fault, through the status block's test knob (word
21): a fused decode launch in which one CTA does not arrive at the first
grid barrier, so that every CTA's wait on it runs out of a 1 ms budget; and
expert GEMMs in which one CTA issues no weight copies, so that its dequant
warps' waits run out of a 1 ms budget while its other roles wind down.  Each time the status must say
MOE_ERR_TIMEOUT, the call must come back long before the 2 s default, and
the next call on the same workspace (status block cleared) must be exact.
"""
import time

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

WAIT_LIMIT_WORD = 20
TEST_KNOB_WORD = 21


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
    d = dict(name=name, T=64, H=512, E=16, k=2, I=256, has_shared=True, wfmt=synth.WFMT_INT4_SYM,
             G=64, wr_std=0.05, zipf_s=0.0, seed=31)
    d.update(kw)
    return synth.LayerConfig(**d)


def test_decode_lost_barrier_arrival_times_out(dev):
    import quantized_moe_expert_warp_b200 as mq
    from quantized_moe_expert_warp_b200.host import upload_layer, x_to_device
    cfg = small_cfg("decode_budget", T=4, E=8, k=2)
    layer = synth.make_layer(cfg)
    packed = upload_layer(layer, dev)
    x = x_to_device(layer["x"], dev)
    n = mq.moe_layer_decode_workspace_size(cfg, cfg.T)
    assert n > 0
    ws = torch.zeros(n, dtype=torch.uint8, device=dev)
    y_ref = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)
    mq.moe_layer_decode(packed, x, cfg.T, y_ref, ws, n)
    assert mq.moe_read_status(ws) == (0, 0)

    words = ws[:256].view(torch.int32)
    words[WAIT_LIMIT_WORD] = 1000     # 1 ms
    words[TEST_KNOB_WORD] = 3         # CTA 2 never arrives at the first barrier
    y = torch.empty_like(y_ref)
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    mq.moe_layer_decode(packed, x, cfg.T, y, ws, n)
    status, detail = mq.moe_read_status(ws)   # synchronises, then clears the whole block
    dt = time.perf_counter() - t0
    assert status == mq.MOE_ERR_TIMEOUT and detail == 91, (status, detail)
    assert dt < 1.0, f"the call took {dt:.3f} s: the 1 ms budget was not applied"
    assert int(ws[:256].view(torch.int32).abs().sum().item()) == 0

    mq.moe_layer_decode(packed, x, cfg.T, y, ws, n)
    assert mq.moe_read_status(ws) == (0, 0)
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))


@pytest.mark.parametrize("cfg", [small_cfg("ffn_budget"),
                                 small_cfg("ffn_budget_q4k", H=512, I=256, G=256, wfmt=synth.WFMT_Q4K),
                                 small_cfg("ffn_budget_wide", T=1200, E=4, k=2)],
                         ids=lambda c: c.name)
def test_expert_gemms_run_out_of_budget_cleanly(dev, cfg):
    """Both grouped GEMMs on a valid permutation, first as they are, then
    with CTA 0's weight copies withheld under a 1 ms budget."""
    import quantized_moe_expert_warp_b200 as mq
    from quantized_moe_expert_warp_b200.host import upload_layer, x_to_device
    layer = synth.make_layer(cfg)
    packed = upload_layer(layer, dev)
    x = x_to_device(layer["x"], dev)
    T, H, E, k = cfg.T, cfg.H, cfg.E, cfg.k
    e32 = lambda *s: torch.empty(s, dtype=torch.float32, device=dev)
    i32 = lambda *s: torch.empty(s, dtype=torch.int32, device=dev)
    logits, gl, ids, w = e32(T, E), e32(T), i32(T, k), e32(T, k)
    counts, offsets, ss, dp = i32(E), i32(E + 1), i32(T * k), i32(T * k)
    rn = mq.moe_router_workspace_size(cfg, T)
    rws = torch.zeros(rn, dtype=torch.uint8, device=dev)
    mq.moe_router_logits(packed, x, T, logits, gl, rws, rn)
    mq.moe_route(logits, T, E, k, cfg.renorm, ids, w)
    pn = mq.moe_permute_workspace_size(T, E, k)
    pws = torch.zeros(pn, dtype=torch.uint8, device=dev)
    mq.moe_permute(ids, T, E, k, counts, offsets, ss, dp, pws, pn)
    assert mq.moe_read_status(pws) == (0, 0)

    n = mq.moe_expert_ffn_workspace_size(cfg, T)
    ws = torch.zeros(n, dtype=torch.uint8, device=dev)
    out = lambda: (torch.zeros((T * k, H), dtype=torch.bfloat16, device=dev),
                   torch.zeros((T, H), dtype=torch.bfloat16, device=dev))
    yp_ref, sh_ref = out()
    mq.moe_expert_ffn_q4(packed, x, T, ss, offsets, yp_ref, sh_ref, ws, n)
    assert mq.moe_read_status(ws) == (0, 0)

    words = ws[:256].view(torch.int32)
    words[WAIT_LIMIT_WORD] = 1000     # 1 ms
    words[TEST_KNOB_WORD] = 1         # CTA 0 issues no weight copies: its dequant waits run out
    yp, sh = out()
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    mq.moe_expert_ffn_q4(packed, x, T, ss, offsets, yp, sh, ws, n)
    status, _ = mq.moe_read_status(ws)
    dt = time.perf_counter() - t0
    assert status == mq.MOE_ERR_TIMEOUT
    assert dt < 1.0, f"the call took {dt:.3f} s"

    mq.moe_expert_ffn_q4(packed, x, T, ss, offsets, yp, sh, ws, n)
    assert mq.moe_read_status(ws) == (0, 0)
    assert torch.equal(yp.view(torch.int16), yp_ref.view(torch.int16))
    assert torch.equal(sh.view(torch.int16), sh_ref.view(torch.int16))
