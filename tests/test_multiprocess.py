"""The N > 1 path on CPU: replicas share weights and split tokens, timing is
the max over ranks, and the reference arm prints one line from rank 0 only.

The layer shards by token with no exchange between ranks, so the only
collectives are the barrier and the max-over-ranks reduction of the step
time; both run here over gloo with two processes."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        out[rank] = bench.max_over_ranks(1.5 + rank, world, "cpu")
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_barrier_gloo():
    import torch.multiprocessing as mp
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        assert dict(out) == {0: 2.5, 1: 2.5}


def test_replicas_share_weights_and_split_tokens():
    cfg = synth.get_config("tiny_t64")
    a = synth.make_layer(bench.replica_config(cfg, 0))
    b = synth.make_layer(bench.replica_config(cfg, 1))
    assert bench.replica_config(cfg, 0) == cfg
    for key in ("router_w", "gu_nib", "gu_scale", "dn_nib", "dn_scale"):
        assert np.array_equal(a[key], b[key]), key
    assert a["x"].shape == b["x"].shape and not np.array_equal(a["x"], b["x"])


def test_reference_arm_under_torchrun_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--config", "tiny_t64", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--ref-sample", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
