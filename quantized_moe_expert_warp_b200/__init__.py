"""Thin Python binding of libmoeq4 (4-bit quantized MoE expert layer, B200).

Every function here only marshals arguments for the C ABI declared in
``include/moeq4.h``; all computation runs in the library's CUDA kernels.
Tensors are torch tensors on the CUDA device (torch supplies device memory
and streams) or raw integer device addresses.  The library must be built
(``python -m quantized_moe_expert_warp_b200.build``); importing the
binding without it raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes as C
import os

__all__ = [
    "MoeError", "Config", "lib", "moe_version", "moe_last_error", "moe_packed_sizes", "moe_pack_weights",
    "moe_dequant_export", "moe_router_workspace_size", "moe_router_logits", "moe_route", "moe_permute_workspace_size", "moe_permute",
    "moe_expert_ffn_workspace_size", "moe_expert_ffn_q4", "moe_combine", "moe_gather_rows", "moe_layer_workspace_size",
    "moe_layer_forward", "moe_layer_forward_chunked", "moe_layer_decode_workspace_size", "moe_layer_decode", "moe_read_status", "moe_kernel_launches", "moe_expert_gate_up_q4", "moe_expert_down_q4",
    "moe_permute_noalloc", "PackedLayer", "WFMT_INT4_SYM", "WFMT_Q4K", "WFMT_INT4_ASYM", "WFMT_INT4_SYM_F16",
    "LIB_PATH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoeq4.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_CUDA = -3
MOE_ERR_TIMEOUT = -4
MOE_ERR_WORKSPACE = -5
WFMT_INT4_SYM = 0
WFMT_Q4K = 1
WFMT_INT4_ASYM = 2
WFMT_INT4_SYM_F16 = 3

_NAMES = {0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_CUDA",
          -4: "MOE_ERR_TIMEOUT", -5: "MOE_ERR_WORKSPACE"}


class MoeError(RuntimeError):
    def __init__(self, code, fn, msg):
        super().__init__(f"{fn}: {_NAMES.get(code, code)}: {msg}")
        self.code = code


class Config(C.Structure):
    _fields_ = [("H", C.c_int32), ("I", C.c_int32), ("E", C.c_int32), ("k", C.c_int32), ("G", C.c_int32),
                ("has_shared", C.c_int32), ("renorm", C.c_int32), ("wfmt", C.c_int32)]

    @classmethod
    def of(cls, cfg) -> "Config":
        """From any object with H, I, E, k, G, has_shared, renorm, wfmt attributes."""
        return cls(cfg.H, cfg.I, cfg.E, cfg.k, cfg.G, int(cfg.has_shared), int(getattr(cfg, "renorm", True)),
                   cfg.wfmt)


class Layer(C.Structure):
    _fields_ = [("cfg", Config), ("router_w", C.c_void_p), ("router_bias", C.c_void_p),
                ("shared_gate", C.c_void_p), ("gu_q", C.c_void_p), ("gu_meta", C.c_void_p),
                ("dn_q", C.c_void_p), ("dn_meta", C.c_void_p)]


class Debug(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("logits", "gate_logit", "topk_ids", "topk_w", "counts", "offsets",
                                         "sorted_slot", "dest_pos", "override_ids", "override_w")]


_lib = None


def lib():
    """Load libmoeq4.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m quantized_moe_expert_warp_b200.build`")
        L = C.CDLL(LIB_PATH)
        vp, i32, sz = C.c_void_p, C.c_int, C.c_size_t
        sig = {
            "moe_last_error": (C.c_char_p, []),
            "moe_version": (i32, []),
            "moe_kernel_launches": (C.c_uint64, []),
            "moe_expert_gate_up_q4": (i32, [vp, vp, i32, vp, vp, vp, vp, sz, vp]),
            "moe_expert_down_q4": (i32, [vp, vp, i32, vp, vp, vp, vp, sz, vp]),
            "moe_packed_sizes": (i32, [vp, vp, vp, vp, vp]),
            "moe_pack_weights": (i32, [vp] * 10),
            "moe_dequant_export": (i32, [vp, vp, vp, i32, i32, vp, vp, vp]),
            "moe_router_workspace_size": (C.c_size_t, [vp, i32]),
            "moe_router_logits": (i32, [vp, vp, i32, vp, vp, vp, C.c_size_t, vp]),
            "moe_route": (i32, [vp, i32, i32, i32, i32, vp, vp, vp]),
            "moe_permute_workspace_size": (sz, [i32, i32, i32]),
            "moe_permute": (i32, [vp, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp]),
            "moe_permute_noalloc": (i32, [vp, i32, i32, i32, vp, vp, vp, vp, vp]),
            "moe_expert_ffn_workspace_size": (sz, [vp, i32]),
            "moe_expert_ffn_q4": (i32, [vp, vp, i32, vp, vp, vp, vp, vp, sz, vp]),
            "moe_combine": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, vp, vp]),
            "moe_gather_rows": (i32, [vp, vp, i32, i32, i32, vp, vp]),
            "moe_layer_workspace_size": (sz, [vp, i32]),
            "moe_layer_forward": (i32, [vp, vp, i32, vp, vp, sz, vp, vp]),
            "moe_layer_forward_chunked": (i32, [vp, vp, i32, vp, i32, vp, sz, vp]),
            "moe_layer_decode_workspace_size": (sz, [vp, i32]),
            "moe_layer_decode": (i32, [vp, vp, i32, vp, vp, sz, vp, vp]),
            "moe_read_status": (i32, [vp, vp, i32, vp, vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(t):
    """Device address of a torch tensor / int / None.

    A tensor must be a dense CUDA tensor: the kernels take bare addresses
    with the row-major layouts of moeq4.h, so a host tensor or a strided
    view is refused here rather than read wrongly on the device."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError(f"expected a CUDA tensor, got one on {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"expected a contiguous tensor, got strides {tuple(t.stride())}")
    return t.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _call(name, *args):
    rc = getattr(lib(), name)(*args)
    if rc != MOE_OK:
        raise MoeError(rc, name, lib().moe_last_error().decode())
    return rc


def moe_version() -> int:
    return lib().moe_version()


def moe_kernel_launches() -> int:
    return lib().moe_kernel_launches()


def moe_expert_gate_up_q4(layer: "PackedLayer", x, T, sorted_slot, offsets, h, ws, ws_bytes, stream=None):
    _call("moe_expert_gate_up_q4", C.byref(layer.c_layer), _ptr(x), T, _ptr(sorted_slot), _ptr(offsets),
          _ptr(h), _ptr(ws), ws_bytes, _stream(stream))


def moe_expert_down_q4(layer: "PackedLayer", h, T, offsets, y_perm, shared_out, ws, ws_bytes, stream=None):
    _call("moe_expert_down_q4", C.byref(layer.c_layer), _ptr(h), T, _ptr(offsets), _ptr(y_perm),
          _ptr(shared_out), _ptr(ws), ws_bytes, _stream(stream))


def moe_last_error() -> str:
    return lib().moe_last_error().decode()


def moe_packed_sizes(cfg):
    c = Config.of(cfg)
    out = [C.c_size_t() for _ in range(4)]
    _call("moe_packed_sizes", C.byref(c), *[C.byref(o) for o in out])
    return tuple(o.value for o in out)


def moe_pack_weights(cfg, gu_canon, gu_scale, dn_canon, dn_scale, gu_q, gu_meta, dn_q, dn_meta, stream=None):
    c = Config.of(cfg)
    _call("moe_pack_weights", C.byref(c), _ptr(gu_canon), _ptr(gu_scale), _ptr(dn_canon), _ptr(dn_scale),
          _ptr(gu_q), _ptr(gu_meta), _ptr(dn_q), _ptr(dn_meta), _stream(stream))


def moe_dequant_export(cfg, q, meta, which, expert, out_f32, out_bf16=None, stream=None):
    c = Config.of(cfg)
    _call("moe_dequant_export", C.byref(c), _ptr(q), _ptr(meta), which, expert, _ptr(out_f32), _ptr(out_bf16),
          _stream(stream))


def moe_router_workspace_size(cfg, T) -> int:
    c = Config.of(cfg)
    return lib().moe_router_workspace_size(C.byref(c), T)


def moe_router_logits(layer: "PackedLayer", x, T, logits, gate_logit=None, ws=None, ws_bytes=0, stream=None):
    _call("moe_router_logits", C.byref(layer.c_layer), _ptr(x), T, _ptr(logits), _ptr(gate_logit), _ptr(ws),
          ws_bytes, _stream(stream))


def moe_route(logits, T, E, k, renorm, topk_ids, topk_w, stream=None):
    _call("moe_route", _ptr(logits), T, E, k, int(renorm), _ptr(topk_ids), _ptr(topk_w), _stream(stream))


def moe_permute_workspace_size(T, E, k) -> int:
    return lib().moe_permute_workspace_size(T, E, k)


def moe_permute(topk_ids, T, E, k, counts, offsets, sorted_slot, dest_pos, ws, ws_bytes, stream=None):
    _call("moe_permute", _ptr(topk_ids), T, E, k, _ptr(counts), _ptr(offsets), _ptr(sorted_slot),
          _ptr(dest_pos), _ptr(ws), ws_bytes, _stream(stream))


def moe_permute_noalloc(topk_ids, T, E, k, counts, offsets, sorted_slot, dest_pos, stream=None):
    """moe_permute with the library's built-in scratch array (no workspace; E <= 1024)."""
    _call("moe_permute_noalloc", _ptr(topk_ids), T, E, k, _ptr(counts), _ptr(offsets), _ptr(sorted_slot),
          _ptr(dest_pos), _stream(stream))


def moe_expert_ffn_workspace_size(cfg, T) -> int:
    c = Config.of(cfg)
    return lib().moe_expert_ffn_workspace_size(C.byref(c), T)


def moe_expert_ffn_q4(layer: "PackedLayer", x, T, sorted_slot, offsets, y_perm, shared_out, ws, ws_bytes,
                      stream=None):
    _call("moe_expert_ffn_q4", C.byref(layer.c_layer), _ptr(x), T, _ptr(sorted_slot), _ptr(offsets),
          _ptr(y_perm), _ptr(shared_out), _ptr(ws), ws_bytes, _stream(stream))


def moe_combine(y_perm, dest_pos, topk_w, shared_out, shared_gate_logit, T, H, k, y, stream=None):
    _call("moe_combine", _ptr(y_perm), _ptr(dest_pos), _ptr(topk_w), _ptr(shared_out),
          _ptr(shared_gate_logit), T, H, k, _ptr(y), _stream(stream))


def moe_gather_rows(x, index, rows, k, H, out, stream=None):
    _call("moe_gather_rows", _ptr(x), _ptr(index), rows, k, H, _ptr(out), _stream(stream))


def moe_layer_workspace_size(cfg, T_max) -> int:
    c = Config.of(cfg)
    return lib().moe_layer_workspace_size(C.byref(c), T_max)


def moe_layer_forward(layer: "PackedLayer", x, T, y, ws, ws_bytes, stream=None, debug: dict | None = None):
    dbg = None
    if debug:
        dbg = Debug(**{k: _ptr(v) for k, v in debug.items()})
    _call("moe_layer_forward", C.byref(layer.c_layer), _ptr(x), T, _ptr(y), _ptr(ws), ws_bytes,
          _stream(stream), C.byref(dbg) if dbg is not None else None)


def moe_layer_forward_chunked(layer: "PackedLayer", x, T, y, chunk, ws, ws_bytes, stream=None):
    _call("moe_layer_forward_chunked", C.byref(layer.c_layer), _ptr(x), T, _ptr(y), int(chunk), _ptr(ws), ws_bytes,
          _stream(stream))


def moe_layer_decode_workspace_size(cfg, T) -> int:
    """0 when the fused decode kernel does not take this shape or T (> 8)."""
    c = Config.of(cfg)
    return lib().moe_layer_decode_workspace_size(C.byref(c), T)


def moe_layer_decode(layer: "PackedLayer", x, T, y, ws, ws_bytes, stream=None, debug: dict | None = None):
    dbg = None
    if debug:
        dbg = Debug(**{k: _ptr(v) for k, v in debug.items()})
    _call("moe_layer_decode", C.byref(layer.c_layer), _ptr(x), T, _ptr(y), _ptr(ws), ws_bytes, _stream(stream),
          C.byref(dbg) if dbg is not None else None)


def moe_read_status(ws, stream=None, clear=True):
    st, det = C.c_int(), C.c_int()
    _call("moe_read_status", _ptr(ws), _stream(stream), int(clear), C.byref(st), C.byref(det))
    return st.value, det.value


class PackedLayer:
    """Device-resident layer weights in the kernel layout.

    Built from canonical weights (torch uint8 / uint16 / fp32 tensors on the
    device, layouts as in moeq4.h) with ``moe_pack_weights``; holds the
    ``moe_layer_t`` handed to the C ABI.
    """

    def __init__(self, cfg, router_w, router_bias, shared_gate, gu_canon, gu_scale, dn_canon, dn_scale,
                 stream=None):
        import torch
        self.cfg = cfg
        dev = router_w.device
        sizes = moe_packed_sizes(cfg)
        self.gu_q, self.gu_meta, self.dn_q, self.dn_meta = (
            torch.empty(n, dtype=torch.uint8, device=dev) for n in sizes)
        moe_pack_weights(cfg, gu_canon, gu_scale, dn_canon, dn_scale, self.gu_q, self.gu_meta, self.dn_q,
                         self.dn_meta, stream)
        self.router_w = router_w.contiguous()
        self.router_bias = None if router_bias is None else router_bias.contiguous()
        self.shared_gate = None if shared_gate is None else shared_gate.contiguous()
        self.c_layer = Layer(Config.of(cfg), _ptr(self.router_w), _ptr(self.router_bias),
                             _ptr(self.shared_gate), _ptr(self.gu_q), _ptr(self.gu_meta), _ptr(self.dn_q),
                             _ptr(self.dn_meta))

    def weight_bytes(self) -> int:
        return sum(t.numel() for t in (self.gu_q, self.gu_meta, self.dn_q, self.dn_meta))
