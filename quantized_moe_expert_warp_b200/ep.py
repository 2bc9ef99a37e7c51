"""Expert-parallel MoE layer: the experts sharded over the ranks of a
process group (one process per GPU), the tokens of each rank sent to the
ranks that own their experts and the results sent back.

The hipfire 0.4.3 benchmarks run the A3B layer on one card; the only
multi-card layout on the pages is a split of whole layers over two GPUs
(the Qwen3.5 Apple Silicon vs ROCm/Vulkan write-up, methodology).  This
module is the expert-sharded layout of the same layer:

  rank r owns the E / W routed experts [r E/W, (r+1) E/W) and a copy of
  the router and of the shared expert.  Per call, on its own T tokens:

  1. router logits, top-k routing and the permutation by expert
     (moe_router_logits, moe_route, moe_permute): counts[E], offsets,
     sorted_slot, dest_pos;
  2. the tokens' rows in permuted order (moe_gather_rows); the rows of
     the experts of rank d are one contiguous block, sent to d;
  3. an all-to-all of the per-expert counts, then of the rows
     (torch.distributed.all_to_all_single; NCCL on GPUs): rank r receives,
     from every rank s, a block of rows ordered by r's local expert;
  4. the received rows in expert-major order (expert, then source rank)
     feed the grouped expert FFN on r's experts (moe_expert_ffn_q4 with
     k = 1, the receive order as sorted_slot);
  5. the results go back in the order they came (the inverse order), and
     a second all-to-all returns each rank its rows in its own permuted
     order: its y_perm;
  6. the shared expert on the rank's own tokens and the weighted combine
     (moe_combine), exactly as in the one-GPU layer.

The exchange is plain NCCL all-to-all of device buffers; no kernel of this
library reads another GPU's memory.  The planning (steps 2-5) is integer
bookkeeping on the host, in the functions below, so that it can be checked
on CPU ranks.
"""
from __future__ import annotations

import numpy as np


def owned_experts(E: int, world: int, rank: int) -> range:
    """The routed experts of a rank: a contiguous block of E / world."""
    if E % world:
        raise ValueError(f"E = {E} is not a multiple of the world size {world}")
    n = E // world
    return range(rank * n, (rank + 1) * n)


def send_counts(counts: np.ndarray, world: int) -> np.ndarray:
    """Rows this rank sends to each rank: its permuted rows of that rank's
    experts (one contiguous block per destination, in rank order)."""
    counts = np.asarray(counts, np.int64)
    return counts.reshape(world, -1).sum(axis=1)


def receive_order(recv_cnt: np.ndarray):
    """Expert-major order of the received rows.

    recv_cnt[s, l]: rows that rank s sent for this rank's local expert l
    (the received rows are rank s's block after rank s - 1's, each block
    ordered by l).  Returns (order, offsets): order[q] is the received row
    that comes q-th when the rows are ordered by local expert, then by
    source rank, then as they arrived; offsets[l] is the first of expert
    l's rows in that order (offsets[-1] = all rows).
    """
    recv_cnt = np.asarray(recv_cnt, np.int64)
    W, El = recv_cnt.shape
    block_start = np.concatenate([[0], np.cumsum(recv_cnt.sum(axis=1))[:-1]])
    in_block = np.concatenate([np.zeros((W, 1), np.int64), np.cumsum(recv_cnt, axis=1)[:, :-1]], axis=1)
    order = []
    for l in range(El):
        for s in range(W):
            a = block_start[s] + in_block[s, l]
            order.append(np.arange(a, a + recv_cnt[s, l], dtype=np.int64))
    order = np.concatenate(order) if order else np.zeros(0, np.int64)
    per_expert = recv_cnt.sum(axis=0)
    offsets = np.concatenate([[0], np.cumsum(per_expert)])
    return order.astype(np.int32), offsets.astype(np.int32)


def inverse(order: np.ndarray) -> np.ndarray:
    inv = np.empty_like(order)
    inv[order] = np.arange(len(order), dtype=order.dtype)
    return inv


def exchange(tensor_out, tensor_in, out_splits, in_splits, group=None):
    """All-to-all of rows (the first dimension), split sizes in rows."""
    import torch.distributed as dist
    dist.all_to_all_single(tensor_out, tensor_in, [int(v) for v in out_splits], [int(v) for v in in_splits],
                           group=group)


class ExpertParallelLayer:
    """One rank's part of the expert-parallel layer (see the module doc).

    ``layer`` is the canonical layer dictionary of ``synth.make_layer``
    (all experts); the rank packs the router, its own experts and the
    shared expert.  Device memory comes from torch; the computation runs in
    the library's kernels and NCCL.
    """

    def __init__(self, layer: dict, rank: int, world: int, device, group=None):
        import torch
        from . import Config, Layer, PackedLayer, WFMT_Q4K
        from .host import to_device
        self.cfg = cfg = layer["cfg"]
        self.rank, self.world, self.device, self.group = rank, world, device, group
        self.own = owned_experts(cfg.E, world, rank)
        El = len(self.own)
        fmt_keys = ("gu_q4k", "dn_q4k") if cfg.wfmt == WFMT_Q4K else ("gu_nib", "gu_scale", "dn_nib", "dn_scale")

        def sub_layer(experts, name):
            sub_cfg = cfg.with_(name=name, E=len(experts), k=1, has_shared=False, zipf_s=0.0)
            d = {"cfg": sub_cfg, "router_w": np.zeros((len(experts), cfg.H), np.float32), "router_bias": None,
                 "shared_gate": None}
            for key in fmt_keys:
                d[key] = layer[key][list(experts)]
            return sub_cfg, d

        def pack(sub_cfg, d):
            rw = to_device(d["router_w"], device)
            if sub_cfg.wfmt == WFMT_Q4K:
                gu, gs, dn, ds = to_device(d["gu_q4k"], device), None, to_device(d["dn_q4k"], device), None
            else:
                gu, dn = to_device(d["gu_nib"], device), to_device(d["dn_nib"], device)
                gs = to_device(d["gu_scale"].view(np.int16), device)
                ds = to_device(d["dn_scale"].view(np.int16), device)
            p = PackedLayer(sub_cfg, rw, None, None, gu, gs, dn, ds)
            torch.cuda.current_stream(device).synchronize()
            return p

        self.local_cfg, d = sub_layer(self.own, f"{cfg.name}_rank{rank}")
        self.local = pack(self.local_cfg, d)
        self.shared = None
        if cfg.has_shared:
            self.shared_cfg, d = sub_layer([cfg.E], f"{cfg.name}_shared")
            self.shared = pack(self.shared_cfg, d)
        # routing: the full router (and shared gate) with this rank's expert
        # buffers in the layer record; the router kernels read only the former
        self.router_w = to_device(layer["router_w"].astype(np.float32), device)
        self.router_b = (None if layer.get("router_bias") is None
                         else to_device(layer["router_bias"].astype(np.float32), device))
        self.shared_gate = (None if layer.get("shared_gate") is None
                            else to_device(layer["shared_gate"].astype(np.float32), device))
        lc = self.local.c_layer
        self.route_layer = Layer(Config.of(cfg), self.router_w.data_ptr(),
                                 self.router_b.data_ptr() if self.router_b is not None else None,
                                 self.shared_gate.data_ptr() if self.shared_gate is not None else None,
                                 lc.gu_q, lc.gu_meta, lc.dn_q, lc.dn_meta)
        self.El = El

    # ------------------------------------------------------------ phases

    def dispatch(self, x, T: int, stream=None) -> dict:
        """Steps 1-2: routing, the permutation and the rows in permuted
        order; returns the state with the per-expert counts (host) and the
        rows to send per rank."""
        import ctypes as C
        import torch
        from . import (_call, _ptr, _stream, moe_gather_rows, moe_permute, moe_permute_workspace_size, moe_route,
                       moe_router_workspace_size, moe_read_status)
        cfg, dev = self.cfg, self.device
        H, E, k = cfg.H, cfg.E, cfg.k
        e32 = lambda *s: torch.empty(s, dtype=torch.float32, device=dev)
        i32 = lambda *s: torch.empty(s, dtype=torch.int32, device=dev)
        st = {"T": T, "logits": e32(T, E), "gl": e32(T), "ids": i32(T, k), "w": e32(T, k), "counts": i32(E),
              "offsets": i32(E + 1), "ss": i32(T * k), "dp": i32(T * k), "x": x}
        rn = moe_router_workspace_size(cfg, T)
        rws = torch.zeros(rn, dtype=torch.uint8, device=dev)
        _call("moe_router_logits", C.byref(self.route_layer), _ptr(x), T, _ptr(st["logits"]),
              _ptr(st["gl"]) if cfg.has_shared else None, _ptr(rws), rn, _stream(stream))
        moe_route(st["logits"], T, E, k, cfg.renorm, st["ids"], st["w"], stream)
        pn = moe_permute_workspace_size(T, E, k)
        pws = torch.zeros(pn, dtype=torch.uint8, device=dev)
        moe_permute(st["ids"], T, E, k, st["counts"], st["offsets"], st["ss"], st["dp"], pws, pn, stream)
        st["x_perm"] = torch.empty((max(T * k, 1), H), dtype=torch.bfloat16, device=dev)
        moe_gather_rows(x, st["ss"], T * k, k, H, st["x_perm"], stream)
        code, det = moe_read_status(pws, stream)
        if code != 0:
            raise RuntimeError(f"permutation: device status {code} ({det})")
        st["counts_host"] = st["counts"].cpu().numpy().astype(np.int64)
        st["sends"] = send_counts(st["counts_host"], self.world)
        return st

    def compute(self, recv_cnt: np.ndarray, x_recv, stream=None):
        """Step 4 and the first half of step 5: this rank's experts on the
        rows it received (recv_cnt[s, l] rows of rank s for local expert
        l, x_recv the rows in arrival order); returns the results in arrival
        order."""
        import torch
        from . import moe_expert_ffn_q4, moe_expert_ffn_workspace_size, moe_gather_rows, moe_read_status
        dev, H = self.device, self.cfg.H
        R = int(np.asarray(recv_cnt).sum())
        y_back = torch.empty((max(R, 1), H), dtype=torch.bfloat16, device=dev)
        if R == 0:
            return y_back
        order, loc_off = receive_order(recv_cnt)
        y_loc = torch.empty((R, H), dtype=torch.bfloat16, device=dev)
        fn = moe_expert_ffn_workspace_size(self.local_cfg, R)
        fws = torch.zeros(fn, dtype=torch.uint8, device=dev)
        moe_expert_ffn_q4(self.local, x_recv, R, torch.from_numpy(order).to(dev), torch.from_numpy(loc_off).to(dev),
                          y_loc, None, fws, fn, stream)
        code, det = moe_read_status(fws, stream)
        if code != 0:
            raise RuntimeError(f"local experts: device status {code} ({det})")
        moe_gather_rows(y_loc, torch.from_numpy(inverse(order)).to(dev), R, 1, H, y_back, stream)
        return y_back

    def combine(self, st: dict, y_perm, y, stream=None):
        """Step 6: the shared expert on the own tokens and the weighted sum."""
        import torch
        from . import moe_combine, moe_expert_ffn_q4, moe_expert_ffn_workspace_size, moe_read_status
        dev, T, H, k = self.device, st["T"], self.cfg.H, self.cfg.k
        S = None
        if self.shared is not None:
            S = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
            ident = torch.arange(T, dtype=torch.int32, device=dev)
            off_s = torch.tensor([0, T], dtype=torch.int32, device=dev)
            sn = moe_expert_ffn_workspace_size(self.shared_cfg, T)
            sws = torch.zeros(sn, dtype=torch.uint8, device=dev)
            moe_expert_ffn_q4(self.shared, st["x"], T, ident, off_s, S, None, sws, sn, stream)
            code, det = moe_read_status(sws, stream)
            if code != 0:
                raise RuntimeError(f"shared expert: device status {code} ({det})")
        moe_combine(y_perm, st["dp"], st["w"], S, st["gl"] if S is not None else None, T, H, k, y, stream)

    # ------------------------------------------------------------- a call

    def forward(self, x, T: int, y, stream=None) -> dict:
        """y [T, H] bf16 <- the layer on this rank's tokens x [T, H] bf16
        (every rank of the group calls it; the exchanges are collective)."""
        import torch
        W, El, H, k = self.world, self.El, self.cfg.H, self.cfg.k
        st = self.dispatch(x, T, stream)
        sends = st["sends"]
        cnt_in = torch.from_numpy(st["counts_host"]).to(self.device)
        cnt_out = torch.empty(W * El, dtype=torch.int64, device=self.device)
        if W > 1:
            exchange(cnt_out, cnt_in, [El] * W, [El] * W, self.group)
        else:
            cnt_out.copy_(cnt_in)
        recv_cnt = cnt_out.cpu().numpy().reshape(W, El)
        recvs = recv_cnt.sum(axis=1)
        R = int(recvs.sum())
        x_recv = torch.empty((max(R, 1), H), dtype=torch.bfloat16, device=self.device)
        if W > 1:
            exchange(x_recv[:R], st["x_perm"][:T * k], recvs, sends, self.group)
        elif R:
            x_recv[:R].copy_(st["x_perm"][:T * k])
        y_back = self.compute(recv_cnt, x_recv, stream)
        y_perm = torch.empty((max(T * k, 1), H), dtype=torch.bfloat16, device=self.device)
        if W > 1:
            exchange(y_perm[:T * k], y_back[:R], sends, recvs, self.group)
        elif T * k:
            y_perm[:T * k].copy_(y_back[:R])
        self.combine(st, y_perm, y, stream)
        return {"topk_ids": st["ids"], "sends": sends, "recv_cnt": recv_cnt}
