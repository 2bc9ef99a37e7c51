"""Expert-parallel layer: the dispatch and return bookkeeping.

The planning functions are checked against brute force; two gloo ranks on
CPU run the whole exchange (counts, rows out, rows back) through
torch.distributed.all_to_all_single with the experts' outputs computed on
the receiving rank, and each rank's combined output must equal the CPU
oracle's layer on its tokens.  On a GPU the same layer runs through the
library's kernels: as one rank, and as several ranks on one GPU whose
exchanges the test carries out by copying the buffers (no kernel waits on
another rank).
"""
import os
import socket

import numpy as np
import pytest

import oracle
import synth
from quantized_moe_expert_warp_b200 import ep

torch = pytest.importorskip("torch")


def test_send_counts_are_block_sums():
    counts = np.array([3, 0, 5, 1, 2, 2, 0, 7])
    assert ep.send_counts(counts, 2).tolist() == [9, 11]
    assert ep.send_counts(counts, 4).tolist() == [3, 6, 4, 7]
    assert ep.owned_experts(8, 4, 2) == range(4, 6)
    with pytest.raises(ValueError):
        ep.owned_experts(10, 4, 0)


@pytest.mark.parametrize("W,El,seed", [(2, 3, 0), (4, 2, 1), (3, 5, 2), (1, 4, 3)])
def test_receive_order_bruteforce(W, El, seed):
    rng = np.random.default_rng(seed)
    recv_cnt = rng.integers(0, 4, size=(W, El))
    recv_cnt[0, 0] = 0
    # the received rows, tagged (source rank, local expert, position in its run)
    tags = []
    for s in range(W):
        for l in range(El):
            tags += [(s, l, i) for i in range(recv_cnt[s, l])]
    order, offsets = ep.receive_order(recv_cnt)
    assert sorted(order.tolist()) == list(range(len(tags)))
    got = [tags[q] for q in order]
    assert got == sorted(tags, key=lambda t: (t[1], t[0], t[2]))
    assert offsets.tolist() == [0] + np.cumsum(recv_cnt.sum(axis=0)).tolist()
    inv = ep.inverse(order)
    assert np.array_equal(order[inv], np.arange(len(order)))


def _dense(layer):
    """Every expert's weights in fp64 (the oracle's dequantisation)."""
    cfg = layer["cfg"]
    H, I = cfg.H, cfg.I
    gu = [oracle.dequant_int4sym(layer["gu_nib"][e], layer["gu_scale"][e], 2 * I, H, cfg.G) for e in range(cfg.E_total)]
    dn = [oracle.dequant_int4sym(layer["dn_nib"][e], layer["dn_scale"][e], H, I, cfg.G) for e in range(cfg.E_total)]
    return np.stack(gu).astype(np.float64), np.stack(dn).astype(np.float64)


def _ffn(x, gu, dn, I):
    a, u = x @ gu[:I].T, x @ gu[I:].T
    return (a / (1.0 + np.exp(-a)) * u) @ dn.T


def _cfg():
    return synth.LayerConfig(name="ep_check", T=40, H=128, E=8, k=3, I=128, has_shared=True,
                             wfmt=synth.WFMT_INT4_SYM, G=32, wr_std=0.08, zipf_s=0.0, seed=17)


def _rank_layer(cfg, rank):
    return synth.make_layer(cfg.with_(x_stream=101 + rank))


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = _cfg()
        layer = _rank_layer(cfg, rank)
        T, H, E, k, I = cfg.T, cfg.H, cfg.E, cfg.k, cfg.I
        gu, dn = _dense(layer)
        x = synth.bf16_bits_to_f32(layer["x"]).astype(np.float64)
        # steps 1-2 as the oracle defines them: routing, permutation, rows in permuted order
        logits = oracle.router_logits(layer["x"], layer["router_w"], layer["router_bias"])
        ids, w32, w64 = oracle.route(logits, k, True)
        counts, offsets, ss, dp = oracle.permute(ids, E)
        x_perm = x[ss // k]
        sends = ep.send_counts(counts, world)
        El = E // world
        cnt_out = torch.empty(world * El, dtype=torch.int64)
        ep.exchange(cnt_out, torch.from_numpy(counts.astype(np.int64)), [El] * world, [El] * world)
        recv_cnt = cnt_out.numpy().reshape(world, El)
        recvs = recv_cnt.sum(axis=1)
        R = int(recvs.sum())
        x_recv = torch.empty((R, H), dtype=torch.float64)
        ep.exchange(x_recv, torch.from_numpy(x_perm), recvs, sends)
        # step 4: this rank's experts on the rows in expert-major order
        order, loc_off = ep.receive_order(recv_cnt)
        xr = x_recv.numpy()[order]
        y_loc = np.empty_like(xr)
        for l, e in enumerate(ep.owned_experts(E, world, rank)):
            a, b = loc_off[l], loc_off[l + 1]
            y_loc[a:b] = _ffn(xr[a:b], gu[e], dn[e], I)
        # step 5: back in arrival order, back to the ranks
        y_back = y_loc[ep.inverse(order)]
        y_perm = torch.empty((T * k, H), dtype=torch.float64)
        ep.exchange(y_perm, torch.from_numpy(np.ascontiguousarray(y_back)), sends, recvs)
        # step 6: shared expert and the combine (the oracle's combine)
        S = _ffn(x, gu[E], dn[E], I)
        z = x @ layer["shared_gate"].astype(np.float64)
        y = oracle.combine(y_perm.numpy(), dp, w64, S, z)
        ref = oracle.layer_forward(layer)["y"]
        out[rank] = float(np.abs(y - ref).max() / np.abs(ref).max())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("world", [2])
def test_expert_parallel_exchange_gloo_matches_oracle(world):
    import torch.multiprocessing as mp
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        errs = dict(out)
    assert sorted(errs) == list(range(world))
    for r, err in errs.items():
        assert err < 1e-12, (r, err)


# --------------------------------------------------------------------- GPU

@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_moe_expert_warp_b200 as mq
    from quantized_moe_expert_warp_b200 import build
    build.build()
    mq.lib()
    return torch.device("cuda", 0)


def _check(layer, y, ids):
    from gpu_util import compare_layer
    return compare_layer(layer, {"y": y.float().cpu().numpy(), "topk_ids": ids.cpu().numpy()})


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["ep_one_rank", "a3b_t512"])
def test_expert_parallel_one_rank_matches_oracle(dev, name):
    from quantized_moe_expert_warp_b200.host import x_to_device
    cfg = _cfg().with_(T=96) if name == "ep_one_rank" else synth.get_config(name)
    layer = synth.make_layer(cfg)
    rank_layer = ep.ExpertParallelLayer(layer, 0, 1, dev)
    x = x_to_device(layer["x"], dev)
    y = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)
    info = rank_layer.forward(x, cfg.T, y)
    _check(layer, y, info["topk_ids"])


@pytest.mark.gpu
@pytest.mark.parametrize("W", [2, 4])
def test_expert_parallel_ranks_emulated_on_one_gpu(dev, W):
    """W ranks in one process: each rank's dispatch, the all-to-alls done by
    copying the row blocks, each rank's experts, the return, each rank's
    combine; every rank's output against the oracle on its tokens."""
    from quantized_moe_expert_warp_b200.host import x_to_device
    cfg = _cfg().with_(T=120, E=16, k=4)
    layers = [_rank_layer(cfg, r) for r in range(W)]
    ranks = [ep.ExpertParallelLayer(layers[r], r, W, dev) for r in range(W)]
    xs = [x_to_device(layers[r]["x"], dev) for r in range(W)]
    st = [ranks[r].dispatch(xs[r], cfg.T) for r in range(W)]
    El, k, H = cfg.E // W, cfg.k, cfg.H
    # counts: rank r receives rank s's counts of r's experts
    recv_cnt = [np.stack([st[s]["counts_host"][r * El:(r + 1) * El] for s in range(W)]) for r in range(W)]
    # rows: rank s's block for rank r, in source order
    starts = [np.concatenate([[0], np.cumsum(st[s]["sends"])]) for s in range(W)]
    x_recv = [torch.cat([st[s]["x_perm"][starts[s][r]:starts[s][r + 1]] for s in range(W)]) for r in range(W)]
    y_back = [ranks[r].compute(recv_cnt[r], x_recv[r]) for r in range(W)]
    rstarts = [np.concatenate([[0], np.cumsum(recv_cnt[r].sum(axis=1))]) for r in range(W)]
    for r in range(W):
        y_perm = torch.cat([y_back[d][rstarts[d][r]:rstarts[d][r + 1]] for d in range(W)])
        assert y_perm.shape[0] == cfg.T * k
        y = torch.empty((cfg.T, H), dtype=torch.bfloat16, device=dev)
        ranks[r].combine(st[r], y_perm, y)
        _check(layers[r], y, st[r]["ids"])
