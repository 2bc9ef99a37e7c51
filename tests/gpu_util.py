"""Helpers shared by the GPU parity tests: run the library through its C ABI
on seeded inputs and compare with the CPU oracle."""
import numpy as np

import oracle
import synth

# Tolerances for floating-point layer outputs (bf16 activations, fp32 accumulation):
# max |err| <= 2e-2 * max |ref| and relative L2 error <= 5e-3.
MAX_ABS_FRAC = 2e-2
REL_L2 = 5e-3
# Routing near-ties: a token whose GPU top-k ids differ from the oracle's is
# accepted only where the oracle's logits of the swapped ids differ by less
# than this (relative to max(1, |logit|)).
NEAR_TIE = 1e-4


def bf16_to_f32(t):
    """torch bf16 tensor -> numpy fp32."""
    return t.float().cpu().numpy()


def f32_to_bf16_rne(a):
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(a))


def check_close(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = got - ref
    max_err = float(np.abs(err).max()) if err.size else 0.0
    max_ref = float(np.abs(ref).max()) if ref.size else 0.0
    rel = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300)) if ref.size else 0.0
    assert max_err <= MAX_ABS_FRAC * max_ref, f"{what}: max|err| {max_err:.3e} > {MAX_ABS_FRAC} * {max_ref:.3e}"
    assert rel <= REL_L2, f"{what}: relative L2 {rel:.3e} > {REL_L2}"
    return max_err / max(max_ref, 1e-300), rel


def run_layer(layer, device, packed=None, override_ids=None, override_w=None):
    """moe_layer_forward with every debug export; returns numpy arrays."""
    import torch
    import quantized_moe_expert_warp_b200 as mq
    from quantized_moe_expert_warp_b200.host import upload_layer, x_to_device

    cfg = layer["cfg"]
    T, E, k, H = cfg.T, cfg.E, cfg.k, cfg.H
    packed = packed or upload_layer(layer, device)
    x = x_to_device(layer["x"], device)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=device)
    nbytes = mq.moe_layer_workspace_size(cfg, T)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
    dbg = {
        "logits": torch.empty((T, E), dtype=torch.float32, device=device),
        "gate_logit": torch.empty((T,), dtype=torch.float32, device=device),
        "topk_ids": torch.empty((T, k), dtype=torch.int32, device=device),
        "topk_w": torch.empty((T, k), dtype=torch.float32, device=device),
        "counts": torch.empty((E,), dtype=torch.int32, device=device),
        "offsets": torch.empty((E + 1,), dtype=torch.int32, device=device),
        "sorted_slot": torch.empty((T * k,), dtype=torch.int32, device=device),
        "dest_pos": torch.empty((T * k,), dtype=torch.int32, device=device),
    }
    if override_ids is not None:
        dbg["override_ids"] = torch.from_numpy(np.ascontiguousarray(override_ids, np.int32)).to(device)
        dbg["override_w"] = torch.from_numpy(np.ascontiguousarray(override_w, np.float32)).to(device)
    mq.moe_layer_forward(packed, x, T, y, ws, nbytes, debug=dbg)
    status, detail = mq.moe_read_status(ws)
    assert status == 0, f"device status {status} (detail {detail})"
    out = {n: v.cpu().numpy() for n, v in dbg.items()}
    out["y"] = bf16_to_f32(y)
    out["y_bf16"] = y
    return out


def near_tie_tokens(oracle_logits, oracle_ids, gpu_ids, k):
    """Tokens whose GPU ids differ from the oracle's; asserts each is a near-tie.

    At every position j where the ids differ, the oracle's logits of the two
    ids must be within NEAR_TIE (relative to max(1, |logit|)): an order swap
    of two nearly equal logits inside the top k, or a flip across the k-th
    boundary, caused by the GPU's fp32 logits differing in the last bits.
    """
    bad = np.where(np.any(oracle_ids != gpu_ids, axis=1))[0]
    for t in bad:
        L = oracle_logits[t].astype(np.float64)
        for j in np.where(oracle_ids[t] != gpu_ids[t])[0]:
            a, b = L[oracle_ids[t, j]], L[gpu_ids[t, j]]
            assert abs(a - b) < NEAR_TIE * max(1.0, abs(a)), \
                f"token {t} position {j}: ids {oracle_ids[t, j]} vs {gpu_ids[t, j]}, logit gap {abs(a - b):.3e}"
    return bad


def oracle_rows(layer, sample=None, override_ids=None, threads=None):
    """oracle.layer_forward, with a long sample split over threads.

    The oracle is single-threaded C called through ctypes, which releases
    the GIL, so chunks of the sample run in parallel; every chunk routes and
    permutes the whole batch the same way, and the rows are concatenated in
    sample order.
    """
    import concurrent.futures as cf
    import os
    if sample is None and layer["cfg"].T > 64:
        sample = np.arange(layer["cfg"].T)
    if sample is None or len(sample) <= 32:
        return oracle.layer_forward(layer, sample=sample, override_ids=override_ids)
    n = threads or max(1, min(len(os.sched_getaffinity(0)), 32, len(sample) // 16))
    parts = np.array_split(np.asarray(sample), n)
    with cf.ThreadPoolExecutor(n) as ex:
        outs = list(ex.map(lambda s: oracle.layer_forward(layer, sample=s, override_ids=override_ids), parts))
    ref = dict(outs[0])
    ref["y"] = np.concatenate([o["y"] for o in outs])
    return ref


def compare_layer(layer, got, sample=None):
    """Oracle on the same inputs.  Near-tie tokens are re-run with the GPU's
    expert ids only: the oracle weighs those ids itself, from its own
    logits, so no floating-point value of the CUDA path enters the
    reference."""
    cfg = layer["cfg"]
    ref = oracle_rows(layer, sample=sample)
    ties = near_tie_tokens(ref["logits"], ref["ids"], got["topk_ids"], cfg.k)
    if len(ties):
        ids = ref["ids"].copy()
        ids[ties] = got["topk_ids"][ties]
        ref = oracle_rows(layer, sample=sample, override_ids=ids)
    y = got["y"] if sample is None else got["y"][np.asarray(sample)]
    stats = check_close(y, ref["y"], cfg.name)
    return ref, ties, stats
