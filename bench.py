#!/usr/bin/env python
"""Benchmark of the 4-bit quantized MoE expert layer on B200.

Metric: MoE-layer prefill tokens/s (with TFLOP/s and the fraction of the
layer roofline) for one Qwen3.6-35B-A3B-shaped layer: hidden 2048, 256
routed experts, top-8, expert intermediate 512, one sigmoid-gated shared
expert, symmetric int4 weights in groups of 128.  The default workload is
one 8192-token prefill chunk with Zipf(1.1)-skewed expert selection, the
largest single-GPU workload (seeded synthetic bf16 N(0,1) activations and
random weights); at N = 1 the same line also carries the 512-token batch,
the 4096-token Q4_K-style layer and the decode batches of 1, 8 and 32
tokens under "extra_configs".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

One process per GPU (torchrun for N > 1).  Each rank runs its own
replica on its own tokens (the layer shards by token with no exchange), so
the whole-job value is N * T tokens per step ("weak" scaling).  Rank 0
prints one JSON line.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

FLOP_PER_TOKEN_TERMS = "2*k*3*H*I + 2*3*H*I (shared) + 2*H*E (router) + 2*H (shared gate)"


def flops_per_token(cfg) -> int:
    f = 2 * cfg.k * 3 * cfg.H * cfg.I + 2 * cfg.H * cfg.E
    if cfg.has_shared:
        f += 2 * 3 * cfg.H * cfg.I + 2 * cfg.H
    return f


def expert_bytes(cfg) -> tuple:
    """(gate/up, down) algorithmic bytes of one expert: codes + scales / headers."""
    if cfg.wfmt == 1:
        gu = 2 * cfg.I * (cfg.H // 256) * 144
        dn = cfg.H * (cfg.I // 256) * 144
    else:
        mb = 4 if cfg.wfmt == 2 else 2   # bf16 scale (and minimum for int4-asym) per group
        gu = 2 * cfg.I * cfg.H // 2 + 2 * cfg.I * (cfg.H // cfg.G) * mb
        dn = cfg.H * cfg.I // 2 + cfg.H * (cfg.I // cfg.G) * mb
    return gu, dn


WFMT_NAMES = {0: "int4-sym", 1: "q4k", 2: "int4-asym", 3: "int4-sym, fp16 operands"}
L2_BYTES = 126e6   # B200 L2


# The profiled kernels are compiled from these files alone (other
# translation units and the public header's declarations do not change
# their code): the grouped GEMMs, and the fused decode kernel.
GEMM_SOURCES = ("dequant.cuh", "gemm.cu", "down_gemm.cu", "kernels.h", "ptx.cuh")
DECODE_SOURCES = ("decode.cu", "decode.h", "dequant.cuh", "kernels.h", "ptx.cuh", "topk.cuh")


def kernel_source_hash(kernel_tag: str = "gate_up") -> str:
    """Hash of the sources of a profiled kernel (GEMM_SOURCES, or
    DECODE_SOURCES for the fused decode kernel, under csrc/): a committed
    ncu figure counts only while it matches."""
    h = hashlib.sha256()
    for name in DECODE_SOURCES if kernel_tag == "decode" else GEMM_SOURCES:
        with open(os.path.join(ROOT, "quantized_moe_expert_warp_b200", "csrc", name), "rb") as fh:
            h.update(name.encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_tag: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", f"ncu_{kernel_tag}_{workload}.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("source_sha256") != kernel_source_hash(kernel_tag):
        return None
    try:
        return int(float(vals["dram_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML while work runs."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.01):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.ok = False
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def replica_config(cfg, rank: int):
    """Weak-scaling replicas: every rank runs the same layer (same weights)
    on its own T tokens (its own activation stream)."""
    return cfg if rank == 0 else cfg.with_(x_stream=cfg.x_stream + 7919 * rank)


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ oracle arm

def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_sample_rate(layer, n_tokens: int):
    """Time the CPU oracle (as it stands, one thread) on the first n_tokens
    of the batch, run as a batch of their own.  Tokens never interact in the
    layer, so those tokens' outputs are the ones the whole batch would give;
    routing, permutation, expert FFNs and combine all cover just them.
    Returns (tokens/s, seconds)."""
    import oracle
    oracle.build()
    cfg = layer["cfg"]
    n = min(n_tokens, cfg.T)
    sub = dict(layer, cfg=cfg.with_T(n, f"{cfg.name}_first{n}"), x=layer["x"][:n])
    t0 = time.perf_counter()
    oracle.layer_forward(sub)
    dt = time.perf_counter() - t0
    return n / dt, dt


def run_reference(args, cfg, rank, world):
    if rank != 0:
        return
    import synth
    layer = synth.make_layer(cfg)
    n = min(args.ref_sample, cfg.T)
    for _ in range(args.warmup):
        oracle_sample_rate(layer, n)
    secs = 0.0
    for _ in range(args.steps):
        _, dt = oracle_sample_rate(layer, n)
        secs += dt
    value = args.steps * n / secs
    sample = f"first {n} of {cfg.T} tokens per step, run as their own batch (one host thread of {host_cores()})"
    line = {
        "metric": "MoE-layer prefill tokens/s", "impl": "reference", "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights quantised)",
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "k": cfg.k, "I": cfg.I},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "host_cores": host_cores(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------- our arm

def pct(xs, q):
    """q-th percentile (linear interpolation) of a list."""
    return float(np.percentile(np.asarray(xs, np.float64), q))


def load_peaks():
    mp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    peaks = json.load(open(mp)) if os.path.exists(mp) else {}
    hbm, src = peaks.get("hbm_gbs"), "measured"
    if not hbm:
        hbm, src = 6650.0, "fallback"
    tc = peaks.get("bf16_tflops") or 1590.0
    return hbm, tc, src


class Bench:
    """One layer configuration resident on one GPU: weights packed, inputs
    and workspace allocated, the step callable, and its timing."""

    def __init__(self, cfg, dev, stream, rank=0, decode=False):
        import torch
        import synth
        import quantized_moe_expert_warp_b200 as mq
        from quantized_moe_expert_warp_b200.host import upload_layer, x_to_device
        self.torch, self.mq = torch, mq
        self.cfg, self.dev, self.stream = cfg, dev, stream
        self.layer = synth.make_layer(replica_config(cfg, rank))
        self.packed = upload_layer(self.layer, dev)
        T, H = cfg.T, cfg.H
        self.x = x_to_device(self.layer["x"], dev)
        self.y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        self.decode = decode and mq.moe_layer_decode_workspace_size(cfg, T) > 0
        self.call = mq.moe_layer_decode if self.decode else mq.moe_layer_forward
        self.nbytes = (mq.moe_layer_decode_workspace_size(cfg, T) if self.decode
                       else mq.moe_layer_workspace_size(cfg, T))
        self.ws = torch.zeros(self.nbytes, dtype=torch.uint8, device=dev)
        # When one step reads less than twice the L2 (126 MB), L2 is flushed
        # (a 256 MB write) before every timed step, outside its events;
        # otherwise the step's own weights already exceed L2.
        gu_b, dn_b = expert_bytes(cfg)
        self.gu_b, self.dn_b = gu_b, dn_b
        step_bytes_bound = min(T * cfg.k + 1, cfg.E + 1) * (gu_b + dn_b)
        self.flush = (torch.empty(256 << 20, dtype=torch.uint8, device=dev)
                      if step_bytes_bound < 2 * L2_BYTES else None)

    def step(self):
        self.call(self.packed, self.x, self.cfg.T, self.y, self.ws, self.nbytes, self.stream)

    def check_status(self, where):
        st, det = self.mq.moe_read_status(self.ws, self.stream)
        if st != 0:
            raise RuntimeError(f"{self.cfg.name}: device status {st} ({det}) {where}")

    def timed(self, fn, n):
        """Per-step device ms of n calls of fn (CUDA events on the launching
        stream), and the ms from the first call's start to the last one's end
        (no flush: consecutive events; with the flush the steps are timed
        one by one and the total is their sum)."""
        torch = self.torch
        if self.flush is None:
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
            ev[0].record(self.stream)
            for i in range(n):
                fn()
                ev[i + 1].record(self.stream)
            ev[-1].synchronize()
            per = [ev[i].elapsed_time(ev[i + 1]) for i in range(n)]
            return per, ev[0].elapsed_time(ev[-1])
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for i in range(n):
            self.flush.fill_(i & 0xFF)
            pairs[i][0].record(self.stream)
            fn()
            pairs[i][1].record(self.stream)
        pairs[-1][1].synchronize()
        per = [a.elapsed_time(b) for a, b in pairs]
        return per, sum(per)

    def per_kernel(self, steps):
        """Mean device ms of each step of the kernel chain, run one call at a
        time (the same kernels as the fused call) with events between them."""
        torch, mq, cfg = self.torch, self.mq, self.cfg
        T, H, E, k, dev, st, packed, x = cfg.T, cfg.H, cfg.E, cfg.k, self.dev, self.stream, self.packed, self.x
        e32 = lambda *s: torch.empty(s, dtype=torch.float32, device=dev)
        i32 = lambda *s: torch.empty(s, dtype=torch.int32, device=dev)
        logits, gl, ids, tw = e32(T, E), e32(T), i32(T, k), e32(T, k)
        counts, offsets, ss, dp = i32(E), i32(E + 1), i32(T * k), i32(T * k)
        pn = mq.moe_permute_workspace_size(T, E, k)
        pws = torch.zeros(pn, dtype=torch.uint8, device=dev)
        rn = mq.moe_router_workspace_size(cfg, T)
        rws = torch.zeros(rn, dtype=torch.uint8, device=dev)
        fn = mq.moe_expert_ffn_workspace_size(cfg, T)
        fws = torch.zeros(fn, dtype=torch.uint8, device=dev)
        h = torch.empty((T * k + T, cfg.I), dtype=torch.bfloat16, device=dev)
        y_perm = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev)
        sh = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        names = ["router_logits", "route", "permute", "gate_up_gemm", "down_gemm", "combine"]
        calls = [
            lambda: mq.moe_router_logits(packed, x, T, logits, gl, rws, rn, st),
            lambda: mq.moe_route(logits, T, E, k, cfg.renorm, ids, tw, st),
            lambda: mq.moe_permute(ids, T, E, k, counts, offsets, ss, dp, pws, pn, st),
            lambda: mq.moe_expert_gate_up_q4(packed, x, T, ss, offsets, h, fws, fn, st),
            lambda: mq.moe_expert_down_q4(packed, h, T, offsets, y_perm, sh, fws, fn, st),
            lambda: mq.moe_combine(y_perm, dp, tw, sh, gl, T, H, k, y, st),
        ]
        for _ in range(2):
            for c in calls:
                c()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(steps)]
        torch.cuda.synchronize(dev)
        for s in range(steps):
            if self.flush is not None:
                self.flush.fill_(s & 0xFF)
            evs[s][0].record(st)
            for i, c in enumerate(calls):
                c()
                evs[s][i + 1].record(st)
        torch.cuda.synchronize(dev)
        per = {n: statistics.mean(evs[s][i].elapsed_time(evs[s][i + 1]) for s in range(steps))
               for i, n in enumerate(names)}
        touched = int((counts.cpu().numpy() > 0).sum()) + (1 if cfg.has_shared else 0)
        return per, touched

    def rooflines(self, ms_step, per_kernel_ms, touched):
        """The dominant GEMM's roofline (its algorithmic bytes or FLOPs over
        its own time) and the whole layer's (max of FLOPs at the tensor peak
        and bytes at the HBM peak, over the step time)."""
        cfg = self.cfg
        T, H, E = cfg.T, cfg.H, cfg.E
        hbm_peak, tc_peak, peak_src = load_peaks()
        alg = {"gate_up_gemm": touched * self.gu_b + 2 * T * H, "down_gemm": touched * self.dn_b}
        rows = T * cfg.k + (T if cfg.has_shared else 0)
        flops = {"gate_up_gemm": 2.0 * rows * 2 * cfg.I * H, "down_gemm": 2.0 * rows * H * cfg.I}
        dominant = max(("gate_up_gemm", "down_gemm"), key=lambda n: per_kernel_ms[n])
        tag = {"gate_up_gemm": "gate_up", "down_gemm": "down"}[dominant]
        secs = per_kernel_ms[dominant] * 1e-3
        if flops[dominant] / (tc_peak * 1e12) > alg[dominant] / (hbm_peak * 1e9):
            achieved = flops[dominant] / secs / 1e12
            roof = {"bound": "tensor", "kernel": dominant, "achieved": achieved, "peak": tc_peak,
                    "unit": "TFLOP/s", "frac": achieved / tc_peak, "traffic": ncu_traffic(tag, cfg.name),
                    "algorithmic_flops_per_launch": flops[dominant],
                    "algorithmic_bytes_per_launch": alg[dominant]}
        else:
            achieved = alg[dominant] / secs / 1e9
            roof = {"bound": "hbm", "kernel": dominant, "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                    "frac": achieved / hbm_peak, "traffic": ncu_traffic(tag, cfg.name),
                    "algorithmic_bytes_per_launch": alg[dominant]}
        roof.update({"ms_per_launch": per_kernel_ms[dominant], "peak_source": peak_src})
        layer_bytes = touched * (self.gu_b + self.dn_b) + E * H * 4 + 4 * T * H
        fpt = flops_per_token(cfg)
        t_hbm = layer_bytes / (hbm_peak * 1e9)
        t_tc = T * fpt / (tc_peak * 1e12)
        if self.decode:
            # one kernel is the whole step: its algorithmic bytes are the layer's
            achieved = layer_bytes / (ms_step * 1e-3) / 1e9
            roof = {"bound": "hbm", "kernel": "decode_layer", "achieved": achieved, "peak": hbm_peak,
                    "unit": "GB/s", "frac": achieved / hbm_peak, "traffic": ncu_traffic("decode", cfg.name),
                    "algorithmic_bytes_per_launch": layer_bytes, "ms_per_launch": ms_step, "peak_source": peak_src}
        layer_roof = {"bound": "hbm" if t_hbm >= t_tc else "tensor", "roofline_ms": 1e3 * max(t_hbm, t_tc),
                      "frac": 1e3 * max(t_hbm, t_tc) / ms_step, "bytes": layer_bytes, "flops": T * fpt,
                      "hbm_gbs_achieved": layer_bytes / (ms_step * 1e-3) / 1e9,
                      "tflops_achieved": T * fpt / (ms_step * 1e-3) / 1e12}
        return roof, layer_roof

    def l2_note(self, touched):
        mb = touched * (self.gu_b + self.dn_b) / 1e6
        if self.flush is not None:
            return "flushed before each timed step (256 MB write); a step reads %.0f MB of weights" % mb
        return "inputs larger than L2 (a step reads %.0f MB of expert weights)" % mb


def stats_of(per):
    return {"median": statistics.median(per), "p10": pct(per, 10), "p90": pct(per, 90),
            "mean": statistics.mean(per), "n": len(per)}


def extra_config(name, dev, stream, steps, warmup, decode):
    """A shorter measurement of another workload (rank 0, N = 1): per-step
    device time (median, p10, p90), tokens/s at the median, the dominant
    GEMM's and the layer's roofline fractions."""
    import synth
    import torch
    cfg = synth.get_config(name)
    b = Bench(cfg, dev, stream, decode=decode)
    for _ in range(warmup):
        b.step()
    torch.cuda.synchronize(dev)
    b.check_status("after warm-up")
    per, _ = b.timed(b.step, steps)
    b.check_status("in the timed steps")
    med = statistics.median(per)
    kms, touched = b.per_kernel(min(steps, 10))
    roof, layer_roof = b.rooflines(med, kms, touched)
    out = {"T": cfg.T, "weights": WFMT_NAMES[cfg.wfmt], "path": "fused decode kernel" if b.decode else "kernel chain",
           "ms_per_step": stats_of(per), "tokens_per_s": cfg.T / (med * 1e-3),
           "tflops": cfg.T * flops_per_token(cfg) / (med * 1e-3) / 1e12,
           "roofline": roof, "layer_roofline": layer_roof, "per_kernel_ms": kms,
           "experts_touched": touched, "l2": b.l2_note(touched)}
    del b
    torch.cuda.empty_cache()
    return out


DEFAULT_EXTRAS = ("a3b_t512", "a3b_t4096_q4k", "a3b_t8192_zipf_f16", "a3b_decode_t1", "a3b_decode_t8",
                  "a3b_decode_t32")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="a3b_t8192_zipf")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-sample", type=int, default=8, help="tokens per oracle step (reference arm)")
    ap.add_argument("--cpu-sample", type=int, default=256, help="tokens of the CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the other workloads (N = 1 only)")
    ap.add_argument("--profile", action="store_true", help="short run for ncu: no e2e / cpu / extra legs")
    ap.add_argument("--decode", action="store_true", help="T <= 8 through the fused decode kernel")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if not args.profile else args.warmup

    import synth
    rank, world, local = dist_setup()
    cfg = synth.get_config(args.config)

    if args.impl == "reference":
        if world > 1:
            import torch.distributed as dist
            import datetime
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
        run_reference(args, cfg, rank, world)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    import torch
    import quantized_moe_expert_warp_b200 as mq

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    stream = torch.cuda.current_stream(dev)
    # every rank: the same layer weights, its own tokens
    b = Bench(cfg, dev, stream, rank=rank, decode=args.decode)
    T, H = cfg.T, cfg.H

    for _ in range(args.warmup):
        b.step()
    torch.cuda.synchronize(dev)
    b.check_status("after warm-up")

    # ---------------------------------------------------------- timed region
    sampler = ClockSampler(local)
    with sampler:
        barrier(world)
        torch.cuda.synchronize(dev)
        launches0 = mq.moe_kernel_launches()
        per, total_ms = b.timed(b.step, args.steps)
        launches = mq.moe_kernel_launches() - launches0
        torch.cuda.synchronize(dev)
        barrier(world)
        # keep the same work running for a short window so that the clock
        # sampler also sees a sustained load when the timed region is short
        t_end = time.perf_counter() + (0.5 if not args.profile else 0.0)
        while time.perf_counter() < t_end:
            for _ in range(20):
                b.step()
            torch.cuda.synchronize(dev)
    ms = total_ms / args.steps
    ms_max = max_over_ranks(ms, world, dev)
    b.check_status("in the timed region")

    value = world * T / (ms_max * 1e-3)
    fpt = flops_per_token(cfg)
    tflops = value * fpt / 1e12

    per_kernel_ms, touched = b.per_kernel(args.steps)
    roofline, layer_roof = b.rooflines(ms, per_kernel_ms, touched)

    # ------------------------------------------------------------------ e2e
    # Through the public call with host buffers: every step copies its input
    # from pinned host memory and its result back to pinned host memory.  The
    # steps are pipelined the way a serving loop runs them: the copies in and
    # out go on their own streams, two device buffers each, so that step i's
    # copies overlap the layer of its neighbours; the timed region runs from
    # the first copy in to the last copy out.
    e2e = None
    if not args.profile:
        x_host = torch.from_numpy(np.ascontiguousarray(b.layer["x"]).view(np.int16)).pin_memory()
        y_host = [torch.empty((T, H), dtype=torch.int16).pin_memory() for _ in range(2)]
        x_in = [torch.empty((T, H), dtype=torch.int16, device=dev) for _ in range(2)]
        y_out = [torch.empty((T, H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_run(n):
            ev = lambda: torch.cuda.Event(enable_timing=False)
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            start.record(s_in)
            comp_done, out_done = [], []
            for i in range(n):
                j = i % 2
                if i >= 2:
                    s_in.wait_event(comp_done[i - 2])   # x_in[j] is no longer read
                with torch.cuda.stream(s_in):
                    x_in[j].copy_(x_host, non_blocking=True)
                e_in = ev()
                e_in.record(s_in)
                stream.wait_event(e_in)
                if i >= 2:
                    stream.wait_event(out_done[i - 2])   # y_out[j] has been copied out
                b.call(b.packed, x_in[j], T, y_out[j], b.ws, b.nbytes, stream)
                e_c = ev()
                e_c.record(stream)
                comp_done.append(e_c)
                s_out.wait_event(e_c)
                with torch.cuda.stream(s_out):
                    y_host[j].copy_(y_out[j].view(torch.int16), non_blocking=True)
                e_o = ev()
                e_o.record(s_out)
                out_done.append(e_o)
            end.record(s_out)
            end.synchronize()
            return start.elapsed_time(end)

        e2e_run(3)
        torch.cuda.synchronize(dev)
        barrier(world)
        e_total = e2e_run(args.steps)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(e_total / args.steps, world, dev)
        e2e = {"value": world * T / (e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": T * H * 2,
               "d2h_bytes_per_step": T * H * 2, "ms_per_step": e_ms,
               "mode": "pipelined: copies in and out on their own streams overlap the layer (two buffers each)"}

    # ------------------------------------------------ other workloads (N = 1)
    extras = None
    if rank == 0 and world == 1 and not args.profile and not args.no_extras:
        extras = {}
        for name in DEFAULT_EXTRAS:
            if name == cfg.name:
                continue
            extras[name] = extra_config(name, dev, stream, min(args.steps, 30), args.warmup, decode=False)
            if synth.get_config(name).T <= 8:
                extras[name + "_fused"] = extra_config(name, dev, stream, min(args.steps, 30), args.warmup,
                                                       decode=True)

    # ---------------------------------------------------------- cpu baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.profile:
        n = min(args.cpu_sample, T)
        rate, dt = oracle_sample_rate(b.layer, n)
        cpu = {"value": rate, "unit": "tokens/s", "cores": 1, "host_cores": host_cores(), "kind": "oracle",
               "sample": f"first {n} of {T} tokens run as their own batch ({dt:.1f} s on one host thread)"}

    if rank == 0:
        line = {
            "metric": "MoE-layer prefill tokens/s", "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": f"synthetic (seeded N(0,1) bf16 activations; N(0,0.02) weights, {WFMT_NAMES[cfg.wfmt]} quantised)",
            "config": {"workload": cfg.name, "T": T, "H": H, "E": cfg.E, "k": cfg.k, "I": cfg.I,
                       "shared_expert": bool(cfg.has_shared), "weights": WFMT_NAMES[cfg.wfmt],
                       "G": cfg.G, "zipf_s": cfg.zipf_s, "tokens_per_rank": T,
                       "parallelism": f"replicas x{world} (token-sharded)",
                       "path": "fused decode kernel" if b.decode else "kernel chain", "l2": b.l2_note(touched)},
            "ms_per_step_stats": stats_of(per),
            "tflops": tflops, "flop_per_token": fpt,
            "roofline": roofline, "layer_roofline": layer_roof,
            "per_kernel_ms": per_kernel_ms, "composed_ms_per_step": sum(per_kernel_ms.values()),
            "experts_touched": touched,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
            "clocks": sampler.summary(),
            "extra_configs": extras,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
