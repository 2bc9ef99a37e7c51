"""CPU oracle for the 4-bit weight-quantized MoE expert layer.

TEST INFRASTRUCTURE ONLY: the library never imports, links or runs this
package.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA path.

The arithmetic lives in ``moe_oracle.c`` (plain single-threaded C, fp64
sums, one function per step of the layer; see its header for the page
passages each step follows).  This module compiles it with gcc on first
use and wraps it with ctypes for numpy arrays.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

WFMT_INT4_SYM = 0
WFMT_Q4K = 1
WFMT_INT4_ASYM = 2
WFMT_INT4_SYM_F16 = 3   # a GPU operand precision of the int4-sym layer: the same layer here


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so (IEEE arithmetic, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _LayerArgs(C.Structure):
    _fields_ = [
        ("T", C.c_int64), ("H", C.c_int64), ("E", C.c_int64), ("k", C.c_int64), ("I", C.c_int64),
        ("has_shared", C.c_int32), ("wfmt", C.c_int32), ("G", C.c_int32), ("renorm", C.c_int32),
        ("x", C.c_void_p), ("router_w", C.c_void_p), ("router_bias", C.c_void_p),
        ("shared_gate", C.c_void_p), ("gu_q", C.c_void_p), ("gu_scale", C.c_void_p),
        ("dn_q", C.c_void_p), ("dn_scale", C.c_void_p), ("override_ids", C.c_void_p),
        ("override_w", C.c_void_p), ("sample", C.c_void_p), ("n_sample", C.c_int64),
        ("y", C.c_void_p), ("logits", C.c_void_p), ("gate_logit", C.c_void_p), ("ids", C.c_void_p),
        ("w", C.c_void_p), ("counts", C.c_void_p), ("offsets", C.c_void_p),
        ("sorted_slot", C.c_void_p), ("dest_pos", C.c_void_p),
    ]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build())
            i64, vp = C.c_int64, C.c_void_p
            L.oracle_dequant_int4sym.argtypes = [vp, vp, i64, i64, i64, vp]
            L.oracle_dequant_q4k.argtypes = [vp, i64, i64, vp]
            L.oracle_dequant_int4asym.argtypes = [vp, vp, i64, i64, i64, vp]
            L.oracle_router_logits.argtypes = [vp, i64, i64, vp, vp, i64, vp]
            L.oracle_route.argtypes = [vp, i64, i64, i64, C.c_int, vp, vp, vp]
            L.oracle_permute.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp]
            L.oracle_layer_forward.argtypes = [C.POINTER(_LayerArgs)]
            L.oracle_combine.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp]
            _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with status {rc}")


# ------------------------------------------------------------------ steps

def dequant_int4sym(nib, scale, N, K, G) -> np.ndarray:
    nib, scale = _c(nib, np.uint8), _c(scale, np.uint16)
    out = np.empty((N, K), np.float32)
    _check(lib().oracle_dequant_int4sym(_p(nib), _p(scale), N, K, G, _p(out)), "dequant_int4sym")
    return out


def dequant_int4asym(nib, sm, N, K, G) -> np.ndarray:
    """sm: uint16 [N, K/G, 2] bf16 (scale, min) pairs."""
    nib, sm = _c(nib, np.uint8), _c(sm, np.uint16)
    out = np.empty((N, K), np.float32)
    _check(lib().oracle_dequant_int4asym(_p(nib), _p(sm), N, K, G, _p(out)), "dequant_int4asym")
    return out


def dequant_q4k(blocks, N, K) -> np.ndarray:
    blocks = _c(blocks, np.uint8)
    out = np.empty((N, K), np.float32)
    _check(lib().oracle_dequant_q4k(_p(blocks), N, K, _p(out)), "dequant_q4k")
    return out


def router_logits(x_bf16, router_w, bias=None) -> np.ndarray:
    x = _c(x_bf16, np.uint16)
    wr = _c(router_w, np.float32)
    b = _c(bias, np.float32)
    T, H = x.shape
    E = wr.shape[0]
    out = np.empty((T, E), np.float32)
    _check(lib().oracle_router_logits(_p(x), T, H, _p(wr), _p(b), E, _p(out)), "router_logits")
    return out


def route(logits, k, renorm=True):
    """Returns (ids int32 [T,k], w fp32 [T,k], w fp64 [T,k])."""
    L = _c(logits, np.float32)
    T, E = L.shape
    ids = np.empty((T, k), np.int32)
    w32 = np.empty((T, k), np.float32)
    w64 = np.empty((T, k), np.float64)
    _check(lib().oracle_route(_p(L), T, E, k, int(bool(renorm)), _p(ids), _p(w32), _p(w64)), "route")
    return ids, w32, w64


def permute(ids, E):
    """Returns (counts [E], offsets [E+1], sorted_slot [T k], dest_pos [T k])."""
    ids = _c(ids, np.int32)
    T, k = ids.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    ss = np.empty(T * k, np.int32)
    dp = np.empty(T * k, np.int32)
    _check(lib().oracle_permute(_p(ids), T, E, k, _p(counts), _p(offsets), _p(ss), _p(dp)), "permute")
    return counts, offsets, ss, dp


def combine(Y, dest_pos, w, S=None, z=None):
    """y [T, H] fp64 from expert rows Y [T k, H], dest_pos [T k], w [T, k]."""
    Y = _c(Y, np.float64)
    dp = _c(dest_pos, np.int32).reshape(-1)
    w = _c(w, np.float64)
    T, k = w.shape
    H = Y.shape[1]
    S = _c(S, np.float64)
    z = _c(z, np.float64)
    y = np.empty((T, H), np.float64)
    _check(lib().oracle_combine(_p(Y), _p(dp), _p(w), _p(S), _p(z), T, H, k, _p(y)), "combine")
    return y


def layer_forward(layer: dict, sample=None, override_ids=None, override_w=None):
    """Run the whole layer on the arrays of ``synth.make_layer``.

    Returns a dict with ``y`` (fp64 [n_sample or T, H]) and the routing
    intermediates (logits, gate_logit, ids, w, counts, offsets,
    sorted_slot, dest_pos).  ``sample`` lists the tokens whose outputs are
    computed (routing and permutation always cover all T tokens).
    ``override_ids`` replaces the oracle's top-k choice; without
    ``override_w`` the oracle weighs those ids itself from its own logits
    (the same softmax as its routing step).
    """
    cfg = layer["cfg"]
    T, H, E, k, I = cfg.T, cfg.H, cfg.E, cfg.k, cfg.I
    keep = {}

    def arr(name, a, dt):
        a = _c(a, dt)
        keep[name] = a
        return _p(a)

    A = _LayerArgs()
    A.T, A.H, A.E, A.k, A.I = T, H, E, k, I
    wfmt = WFMT_INT4_SYM if cfg.wfmt == WFMT_INT4_SYM_F16 else cfg.wfmt
    A.has_shared, A.wfmt, A.G, A.renorm = int(cfg.has_shared), wfmt, cfg.G, int(cfg.renorm)
    A.x = arr("x", layer["x"], np.uint16)
    A.router_w = arr("wr", layer["router_w"], np.float32)
    A.router_bias = arr("rb", layer.get("router_bias"), np.float32)
    A.shared_gate = arr("sg", layer.get("shared_gate"), np.float32)
    if wfmt in (WFMT_INT4_SYM, WFMT_INT4_ASYM):
        A.gu_q = arr("guq", layer["gu_nib"], np.uint8)
        A.gu_scale = arr("gus", layer["gu_scale"], np.uint16)
        A.dn_q = arr("dnq", layer["dn_nib"], np.uint8)
        A.dn_scale = arr("dns", layer["dn_scale"], np.uint16)
    else:
        A.gu_q = arr("guq", layer["gu_q4k"], np.uint8)
        A.dn_q = arr("dnq", layer["dn_q4k"], np.uint8)
    A.override_ids = arr("oi", override_ids, np.int32)
    A.override_w = arr("ow", override_w, np.float32)
    if sample is not None:
        sample = np.ascontiguousarray(sample, np.int32)
        A.sample = arr("smp", sample, np.int32)
        A.n_sample = len(sample)
        ns = len(sample)
    else:
        ns = T
    out = {
        "y": np.empty((ns, H), np.float64),
        "logits": np.empty((T, E), np.float32),
        "gate_logit": np.zeros(T, np.float64),
        "ids": np.empty((T, k), np.int32),
        "w": np.empty((T, k), np.float32),
        "counts": np.empty(E, np.int32),
        "offsets": np.empty(E + 1, np.int32),
        "sorted_slot": np.empty(T * k, np.int32),
        "dest_pos": np.empty(T * k, np.int32),
    }
    for name in out:
        setattr(A, name, _p(out[name]))
    _check(lib().oracle_layer_forward(C.byref(A)), "layer_forward")
    return out
