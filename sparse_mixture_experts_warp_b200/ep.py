"""Expert parallelism: the MoE layer with its experts spread over G ranks.

"Top-k 路由（Top-k Routing）", section "通訊拓撲：All-to-All": once experts live on different
devices, each device sends every token row to the device holding its expert (dispatch) and
gets the expert outputs back (combine), two All-to-All exchanges per layer whose volume is the
rows that leave the device.  "别只比较 Top-k", "两次 All-to-All 是常见 dispatcher 的前向合同":
this dispatch / combine pair is the usual forward contract around the experts.

Rank r holds the Eg = E / G experts [r Eg, (r+1) Eg) and routes its own batch with the full
(replicated) router.  One layer step per rank:

  1. moe_route + moe_permute over all E experts (the library's kernels): the rows come out
     grouped by expert, so the rows bound for rank r are one contiguous range;
  2. count exchange (All-to-All of Eg ints per peer) and moe_ep_plan on the host (one
     device-to-host read of 2 G Eg ints, the split sizes the row exchange needs);
  3. row exchange (All-to-All-v of the rows) into a source-major receive buffer;
  4. moe_ep_reorder to the expert-major layout, the local grouped GEMMs (moe_expert_up_ws /
     moe_expert_down_ws on Eg groups), moe_ep_reorder back;
  5. the reverse All-to-All-v returns each output row to the slot its row came from, and
     moe_combine / moe_balance_stats finish as on one device.

Every arithmetic step runs in the CUDA library; this module moves buffers and calls the
collectives.  The exchange goes through an `a2a` object: DistAllToAll wraps
torch.distributed.all_to_all_single (NCCL on GPUs, gloo on CPU); LocalAllToAll carries G
logical ranks held by one process on one device (the same data movement as plain device
copies), which is how a single GPU runs the whole exchanged layer.
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import (MoeDesc, _check, _ptr, _stream, desc_of, empty_workspace, layer_views, lib,
               moe_balance_stats, moe_combine, moe_expert_down_ws, moe_expert_up_ws, moe_permute,
               moe_route)

__all__ = ["EpPlan", "ep_plan", "DistAllToAll", "LocalAllToAll", "exchange_counts",
           "exchange_rows", "ep_reorder", "EpRank", "ep_layer_forward"]

_I32P = ctypes.POINTER(ctypes.c_int32)
_I64P = ctypes.POINTER(ctypes.c_int64)


@dataclass
class EpPlan:
    G: int
    Eg: int
    send_rows: list            # rows this rank sends to each peer
    send_offsets: list
    recv_rows: list            # rows it receives from each peer
    recv_offsets: list
    local_offsets: list        # [Eg+1] expert-major layout of the received rows
    block_recv: list           # [G*Eg] block (s, e) start in the receive buffer
    block_local: list          # [G*Eg] its start in the expert-major layout
    block_rows: list
    max_block_rows: int

    @property
    def recv_total(self) -> int:
        return int(sum(self.recv_rows))

    @property
    def send_total(self) -> int:
        return int(sum(self.send_rows))


def _fn(name, args):
    f = getattr(lib(), name)
    f.argtypes = args
    f.restype = ctypes.c_int
    return f


def ep_plan(G: int, Eg: int, rows_send, rows_recv) -> EpPlan:
    """moe_ep_plan on host integer sequences of G*Eg row counts (see include/moe.h)."""
    n = G * Eg
    rs = (ctypes.c_int32 * n)(*[int(v) for v in rows_send])
    rr = (ctypes.c_int32 * n)(*[int(v) for v in rows_recv])
    sr, so, rcv, ro = ((ctypes.c_int64 * G)() for _ in range(4))
    lo = (ctypes.c_int32 * (Eg + 1))()
    br, bl, bn = ((ctypes.c_int64 * n)() for _ in range(3))
    mx = ctypes.c_int64()
    f = _fn("moe_ep_plan", [ctypes.c_int32, ctypes.c_int32, _I32P, _I32P, _I64P, _I64P, _I64P,
                            _I64P, _I32P, _I64P, _I64P, _I64P, _I64P])
    _check("moe_ep_plan", f(G, Eg, rs, rr, sr, so, rcv, ro, lo, br, bl, bn, ctypes.byref(mx)))
    return EpPlan(G, Eg, list(sr), list(so), list(rcv), list(ro), list(lo), list(br), list(bl),
                  list(bn), mx.value)


def ep_reorder(d: MoeDesc, plan: EpPlan, src, dst, to_local: bool = True, stream=None):
    """moe_ep_reorder: receive buffer -> expert-major layout (to_local) or back."""
    dev = src.device
    b_src = plan.block_recv if to_local else plan.block_local
    b_dst = plan.block_local if to_local else plan.block_recv
    arrs = torch.tensor([b_src, b_dst, plan.block_rows], dtype=torch.int64).to(dev)
    f = _fn("moe_ep_reorder", [ctypes.POINTER(MoeDesc), ctypes.c_int32, ctypes.c_void_p,
                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                               ctypes.c_void_p, ctypes.c_void_p])
    _check("moe_ep_reorder", f(ctypes.byref(d), plan.G * plan.Eg, _ptr(arrs[0]), _ptr(arrs[1]),
                               _ptr(arrs[2]), plan.max_block_rows, _ptr(src), _ptr(dst),
                               _stream(stream)))
    return arrs           # keep alive until the stream has consumed the block arrays


class DistAllToAll:
    """All-to-All through torch.distributed (one rank per process)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.G = dist.get_world_size(group)

    def __call__(self, outs, ins, out_splits, in_splits):
        # buffers may carry a spare row (never empty); the exchange covers the split totals
        out = outs[0][:sum(out_splits[0])]
        inp = ins[0][:sum(in_splits[0])]
        self.dist.all_to_all_single(out, inp, list(out_splits[0]), list(in_splits[0]),
                                    group=self.group)


class LocalAllToAll:
    """All-to-All among G logical ranks held by this process (plain tensor copies)."""

    def __init__(self, G: int):
        self.G = G

    def __call__(self, outs, ins, out_splits, in_splits):
        G = self.G
        for s in range(G):
            src_off = 0
            for r in range(G):
                n = in_splits[s][r]
                dst_off = sum(out_splits[r][:s])
                if n:
                    outs[r][dst_off:dst_off + n].copy_(ins[s][src_off:src_off + n])
                src_off += n


def exchange_counts(a2a, rows_send_list, Eg):
    """Count exchange: rank r gets rows_recv[s*Eg + e] = rows_send of rank s for expert
    r*Eg + e.  rows_send_list: per local rank, an int32 tensor [G*Eg]."""
    outs = [torch.empty_like(t) for t in rows_send_list]
    splits = [[Eg] * a2a.G for _ in rows_send_list]
    a2a(outs, rows_send_list, splits, splits)
    return outs


def exchange_rows(a2a, send_list, plans, D, dtype, reverse=False):
    """Row exchange by the plans: dispatch (send buffers -> source-major receive buffers) or,
    with reverse=True, combine (receive-layout buffers -> each rank's original row slots)."""
    if not reverse:
        outs = [torch.empty((max(p.recv_total, 1), D), dtype=dtype, device=t.device)
                for p, t in zip(plans, send_list)]
        a2a(outs, send_list, [p.recv_rows for p in plans], [p.send_rows for p in plans])
    else:
        outs = [torch.empty((max(p.send_total, 1), D), dtype=dtype, device=t.device)
                for p, t in zip(plans, send_list)]
        a2a(outs, send_list, [p.send_rows for p in plans], [p.recv_rows for p in plans])
    return outs


@dataclass
class EpRank:
    """One rank's inputs and outputs: its tokens, the replicated router, its Eg experts."""
    rank: int
    x: torch.Tensor
    Wg: torch.Tensor
    bias: object
    W_gate: object            # [Eg, F, D] (SwiGLU) or None
    W_up: torch.Tensor        # [Eg, F, D]
    W_down: torch.Tensor      # [Eg, D, F]
    out: torch.Tensor         # [T, D]
    ws: object = None
    views: object = None


def ep_layer_forward(w, ranks, a2a, stream=None):
    """The exchanged layer for the ranks this process holds (one for DistAllToAll, all G for
    LocalAllToAll).  `w` is the layer's workload/descriptor source (desc_of(w)); token choice
    without shared experts.  Returns the per-rank plans and the temporaries the enqueued work
    still reads (hold them until the stream has finished)."""
    d = desc_of(w)
    G = a2a.G
    if w.select != "token" or w.n_shared or w.E % G:
        raise ValueError("expert parallelism: token choice, no shared experts, G divides E")
    Eg = w.E // G
    for r in ranks:
        if r.ws is None:
            r.ws = empty_workspace(d, r.x.device)
            r.views = layer_views(d, r.ws)
        v = r.views
        moe_route(d, r.x, r.Wg, r.bias, v["expert_ids"], v["gates"], v["logits"],
                  v["importance"], v["scratch"], stream, entropy=v["entropy"])
        moe_permute(d, v["expert_ids"], r.x, v["x_perm"], v["counts"], v["offsets"],
                    v["row_src"], v["inv"], v["scratch"], stream)
    # kept rows per expert, then the count exchange and the plan (host)
    sends = [(r.views["offsets"][1:] - r.views["offsets"][:-1]).to(torch.int32) for r in ranks]
    recvs = exchange_counts(a2a, sends, Eg)
    plans = [ep_plan(G, Eg, s.tolist(), rv.tolist()) for s, rv in zip(sends, recvs)]
    # dispatch
    send = [r.views["x_perm"][:p.send_total] if p.send_total else r.views["x_perm"][:1]
            for r, p in zip(ranks, plans)]
    recv = exchange_rows(a2a, send, plans, w.D, ranks[0].x.dtype)
    # local experts on the expert-major layout
    y_recv = []
    keep = []
    for r, p, buf in zip(ranks, plans, recv):
        rows = max(p.recv_total, 1)
        dev = buf.device
        loc = torch.empty((rows, w.D), dtype=buf.dtype, device=dev)
        keep.append(ep_reorder(d, p, buf, loc, True, stream))
        off = torch.tensor(p.local_offsets, dtype=torch.int32, device=dev)
        h = torch.empty((rows, w.F), dtype=buf.dtype, device=dev)
        y_loc = torch.empty((rows, w.D), dtype=buf.dtype, device=dev)
        moe_expert_up_ws(d, Eg, w.F, loc, off, r.W_gate, r.W_up, h, None, stream)
        moe_expert_down_ws(d, Eg, w.F, h, off, r.W_down, y_loc, None, stream)
        yr = torch.empty((rows, w.D), dtype=buf.dtype, device=dev)
        keep.append(ep_reorder(d, p, y_loc, yr, False, stream))
        keep.append(off)
        y_recv.append(yr)
    # combine: rows come back to the slots they left from
    back = exchange_rows(a2a, y_recv, plans, w.D, ranks[0].x.dtype, reverse=True)
    for r, yb in zip(ranks, back):
        v = r.views
        moe_combine(d, yb, v["inv"], v["gates"], None, r.out, stream)
        moe_balance_stats(d, v["counts"], v["offsets"], v["importance"], v["f"], v["stats"],
                          stream, entropy=v["entropy"])
    return plans, keep + back
