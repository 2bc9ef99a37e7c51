"""moe_permute_noalloc: the permutation for callers that cannot allocate.

Some integrations have no device memory to give the library when they route
tokens (their allocator is locked, or the host framework forbids cudaMalloc
after start-up).  moe_permute_noalloc keeps its scratch in a fixed array
inside the library instead of a caller workspace.  These tests check that it
returns exactly what moe_permute returns and what the CPU oracle's
permutation defines, on calls in a row with different shapes (the shared
scratch must not leak state between calls), including the largest expert
count its array holds, and that it refuses expert counts beyond it.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes as C

import numpy as np
import pytest

import oracle
import quantized_moe_expert_warp_b200 as mq
from quantized_moe_expert_warp_b200 import build as mqbuild


def test_noalloc_rejects_too_many_experts():
    mqbuild.build()
    L = mq.lib()
    rc = L.moe_permute_noalloc(0x1000, 4, 2048, 2, 0x1000, 0x1000, 0x1000, 0x1000, None)
    assert rc == mq.MOE_ERR_UNSUPPORTED
    assert b"1024" in L.moe_last_error()


def _permute_both(torch, dev, ids_np, E):
    T, k = ids_np.shape
    ids = torch.from_numpy(np.ascontiguousarray(ids_np, np.int32)).to(dev)
    i32 = lambda n: torch.full((max(1, n),), -7, dtype=torch.int32, device=dev)
    ref = [i32(E), i32(E + 1), i32(T * k), i32(T * k)]
    n = mq.moe_permute_workspace_size(T, E, k)
    ws = torch.zeros(n, dtype=torch.uint8, device=dev)
    mq.moe_permute(ids, T, E, k, *ref, ws, n)
    got = [i32(E), i32(E + 1), i32(T * k), i32(T * k)]
    n0 = mq.moe_kernel_launches()
    mq.moe_permute_noalloc(ids, T, E, k, *got)
    assert mq.moe_kernel_launches() - n0 == 2      # histogram and scatter kernels
    torch.cuda.synchronize(dev)
    return [t.cpu().numpy()[:m] for t, m in zip(ref, (E, E + 1, T * k, T * k))], \
        [t.cpu().numpy()[:m] for t, m in zip(got, (E, E + 1, T * k, T * k))]


@pytest.mark.gpu
def test_noalloc_matches_workspace_permute_twice():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mqbuild.build()
    dev = torch.device("cuda", 0)
    rng = np.random.default_rng(2024)
    # first call: a skewed 8192-token, 256-expert, top-8 routing (many empty and big experts)
    p = 1.0 / np.arange(1, 257) ** 1.1
    p /= p.sum()
    ids1 = np.stack([rng.choice(256, size=8, replace=False, p=p) for _ in range(8192)]).astype(np.int32)
    # second call: a different, smaller shape reusing the same built-in scratch
    ids2 = np.stack([rng.permutation(64)[:4] for _ in range(300)]).astype(np.int32)
    # third call: the largest expert count the array holds (E = 1024 fills all
    # of it, and the scatter kernel needs more than 48 KB of shared memory)
    ids3 = np.stack([rng.permutation(1024)[:4] for _ in range(3000)]).astype(np.int32)
    for ids, E in ((ids1, 256), (ids2, 64), (ids3, 1024)):
        ref, got = _permute_both(torch, dev, ids, E)
        want = oracle.permute(ids, E)
        for a, b, c, name in zip(got, ref, want, ("counts", "offsets", "sorted_slot", "dest_pos")):
            assert np.array_equal(a, b), name
            assert np.array_equal(a, c), name
