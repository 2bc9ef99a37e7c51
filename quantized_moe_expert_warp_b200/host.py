"""Host-side marshalling: canonical numpy arrays -> device tensors -> PackedLayer.

Only copies and packs (the packing itself runs in the library's kernels).
The layer dictionary uses the canonical layouts documented in moeq4.h:
``x`` bf16 bits [T, H], ``router_w`` fp32 [E, H], ``router_bias`` [E] or
None, ``shared_gate`` [H] or None, and either ``gu_nib``/``gu_scale``/
``dn_nib``/``dn_scale`` (int4-sym) or ``gu_q4k``/``dn_q4k`` (Q4K).
"""
from __future__ import annotations

import numpy as np

from . import PackedLayer, WFMT_Q4K


def to_device(a, device, dtype=None):
    import torch
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(device)


def upload_layer(layer: dict, device="cuda", stream=None) -> PackedLayer:
    import torch
    cfg = layer["cfg"]
    rw = to_device(layer["router_w"].astype(np.float32), device)
    rb = to_device(None if layer.get("router_bias") is None else layer["router_bias"].astype(np.float32), device)
    sg = to_device(None if layer.get("shared_gate") is None else layer["shared_gate"].astype(np.float32), device)
    if cfg.wfmt == WFMT_Q4K:
        gu, gs = to_device(layer["gu_q4k"], device), None
        dn, ds = to_device(layer["dn_q4k"], device), None
    else:
        gu, gs = to_device(layer["gu_nib"], device), to_device(layer["gu_scale"].view(np.int16), device)
        dn, ds = to_device(layer["dn_nib"], device), to_device(layer["dn_scale"].view(np.int16), device)
    packed = PackedLayer(cfg, rw, rb, sg, gu, gs, dn, ds, stream=stream)
    # the canonical copies are only needed until the pack kernels have run
    torch.cuda.current_stream(device).synchronize() if stream is None else stream.synchronize()
    return packed


def x_to_device(x_bits: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).to(device).view(torch.bfloat16)
