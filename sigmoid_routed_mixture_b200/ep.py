"""Expert-parallel form of the MoE block: ctypes binding of include/srm_ep.h,
the host side of the partition and count exchange, and a driver that runs R
ranks as virtual ranks on one GPU.

The routed experts are split in contiguous ranges over R ranks; the shared
expert stays with every rank for its own tokens.  One step (srm_ep.h lists it
in full): route and permute locally, exchange per-expert counts, plan, dispatch
each routed row to its expert's owner, owners run the grouped GEMMs on what they
received, return each row's weighted output to its source's per-slot buffer,
then each rank runs its shared expert and the fixed-order combine.  The result
equals the single-GPU moe_forward on each rank's tokens, bit for bit.

Argument marshalling and host bookkeeping only: every step of the data path
runs in the library's kernels.  Counts are exchanged with torch.distributed
(all_gather; NCCL on GPUs, gloo on CPU) or, for virtual ranks, stacked on one
device.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import moe

MAX_RANKS = 8
WS_TOKEN_ROWS = 0
WS_SLOT_OUTPUTS = 1


class _Peers(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p * MAX_RANKS)]


_bound = False


def lib():
    """The library with the expert-parallel entry points typed."""
    global _bound
    L = moe.lib()
    if not _bound:
        vp, P = ctypes.c_void_p, ctypes.POINTER
        i32, i64 = ctypes.c_int32, ctypes.c_int64
        L.moe_workspace_offset.restype = ctypes.c_size_t
        L.moe_workspace_offset.argtypes = [P(moe._Cfg), i32]
        L.moe_ep_plan.restype = ctypes.c_int
        L.moe_ep_plan.argtypes = [P(moe._Cfg), i32, i32, P(i32), vp, vp, vp, vp, i64, vp, vp]
        L.moe_ep_dispatch.restype = ctypes.c_int
        L.moe_ep_dispatch.argtypes = [P(moe._Cfg), i32, i32, P(i32), vp, vp, vp, vp, vp, P(_Peers),
                                      P(_Peers), P(_Peers), P(i64), vp, vp]
        L.moe_ep_return.restype = ctypes.c_int
        L.moe_ep_return.argtypes = [P(moe._Cfg), i32, vp, P(_Peers), P(i32), vp, ctypes.c_size_t, vp]
        L.moe_ep_shared.restype = ctypes.c_int
        L.moe_ep_shared.argtypes = [P(moe._Cfg), P(moe._Weights), vp, vp, ctypes.c_size_t, vp]
        _bound = True
    return L


# ------------------------------------------------------------------ host side

def partition(E: int, n_ranks: int) -> list[int]:
    """expert_first: rank r owns routed experts [first[r], first[r+1]),
    contiguous ranges as even as possible (the first E % R ranks one more)."""
    if not 1 <= n_ranks <= min(E, MAX_RANKS):
        raise ValueError("need 1 <= n_ranks <= min(E, %d)" % MAX_RANKS)
    q, r = divmod(E, n_ranks)
    first = [0]
    for k in range(n_ranks):
        first.append(first[-1] + q + (1 if k < r else 0))
    return first


def owner_of(first: list[int], e: int) -> int:
    return max(k for k in range(len(first) - 1) if first[k] <= e)


def plan_host(counts_all: np.ndarray, first: list[int], rank: int):
    """What moe_ep_plan computes, on the host: (dst_row [E], recv_offsets
    [E_r + 2], total).  Receive rows are ordered by expert, then source rank,
    then the source's token order."""
    counts_all = np.asarray(counts_all, dtype=np.int64)
    R, E = counts_all.shape
    tot = counts_all.sum(axis=0)
    start = np.concatenate([[0], np.cumsum(tot)])  # rows of experts [0, g)
    dst_row = np.empty(E, dtype=np.int64)
    for e in range(E):
        o = owner_of(first, e)
        dst_row[e] = start[e] - start[first[o]] + counts_all[:rank, e].sum()
    f0, f1 = first[rank], first[rank + 1]
    total = int(start[f1] - start[f0])
    recv_offsets = np.concatenate([start[f0:f1] - start[f0], [total, total]]).astype(np.int64)
    return dst_row, recv_offsets, total


def exchange_counts(counts_local: torch.Tensor, group=None) -> torch.Tensor:
    """All ranks' per-expert counts, [R][E] int32, on counts_local's device
    (torch.distributed all_gather: NCCL for GPU tensors, gloo for CPU ones)."""
    import torch.distributed as dist

    R = dist.get_world_size(group)
    out = [torch.empty_like(counts_local) for _ in range(R)]
    dist.all_gather(out, counts_local.contiguous(), group=group)
    return torch.stack(out)


# ------------------------------------------------------------------ device calls

def workspace_offset(cfg: moe.Config, region: int) -> int:
    off = lib().moe_workspace_offset(ctypes.byref(cfg.c()), region)
    if off == ctypes.c_size_t(-1).value:
        raise moe.MoeError(1, "moe_workspace_offset")
    return off


def _peers(ptrs):
    p = _Peers()
    for k, v in enumerate(ptrs):
        p.ptr[k] = v
    return p


def _i32(vals):
    return (ctypes.c_int32 * len(vals))(*[int(v) for v in vals])


def plan(cfg: moe.Config, first, rank, counts_all, dst_row, recv_offsets, recv_sorted, ws, stream=None):
    L = lib()
    R = len(first) - 1
    moe._check(L.moe_ep_plan(ctypes.byref(cfg.c()), R, rank, _i32(first), moe._ptr(counts_all),
                             moe._ptr(dst_row), moe._ptr(recv_offsets), moe._ptr(recv_sorted),
                             recv_sorted.numel(), moe._ptr(ws), moe._stream(stream)), "moe_ep_plan")


def dispatch(cfg, first, rank, dst_row, x, gate, offsets, sorted_, recv_x, recv_gate, recv_src, capacity,
             ws, stream=None):
    """recv_x / recv_gate / recv_src: one device address (int) per owner rank."""
    L = lib()
    R = len(first) - 1
    cap = (ctypes.c_int64 * R)(*[int(c) for c in capacity])
    moe._check(L.moe_ep_dispatch(ctypes.byref(cfg.c()), R, rank, _i32(first), moe._ptr(dst_row), moe._ptr(x),
                                 moe._ptr(gate), moe._ptr(offsets), moe._ptr(sorted_),
                                 ctypes.byref(_peers(recv_x)), ctypes.byref(_peers(recv_gate)),
                                 ctypes.byref(_peers(recv_src)), cap, moe._ptr(ws), moe._stream(stream)),
               "moe_ep_dispatch")


def ret(owner_cfg, n_ranks, recv_src, dst_y, dst_rows, owner_ws, stream=None):
    L = lib()
    moe._check(L.moe_ep_return(ctypes.byref(owner_cfg.c()), n_ranks, moe._ptr(recv_src),
                               ctypes.byref(_peers(dst_y)), _i32(dst_rows), moe._ptr(owner_ws),
                               owner_ws.numel(), moe._stream(stream)), "moe_ep_return")


def shared(cfg, w13_block, w2_block, x, ws, stream=None):
    L = lib()
    wt = moe._Weights(w13_block.data_ptr(), w2_block.data_ptr())
    moe._check(L.moe_ep_shared(ctypes.byref(cfg.c()), ctypes.byref(wt), moe._ptr(x), moe._ptr(ws), ws.numel(),
                               moe._stream(stream)), "moe_ep_shared")


# ------------------------------------------------------------------ one rank

class EpRank:
    """The state one rank keeps: its router, its experts' packed weights (its
    routed experts as groups 0 .. E_r - 1 and the shared expert as group E_r),
    a source workspace for its own T tokens and an owner workspace and receive
    buffers sized for every rank's assignments (max_rows)."""

    def __init__(self, cfg: moe.Config, first, rank, w_router, bias, w1, w3, w2, ws1, ws3, ws2, max_rows):
        self.cfg, self.first, self.rank = cfg, list(first), rank
        self.R = len(first) - 1
        f0, f1 = first[rank], first[rank + 1]
        self.E_r = f1 - f0
        dev = w_router.device
        pack_cfg = cfg.replace(E=self.E_r, K=1)  # only the weight shapes matter to packing
        self.w13, self.w2 = moe.pack_weights(pack_cfg, w1[f0:f1].contiguous(), w3[f0:f1].contiguous(),
                                             w2[f0:f1].contiguous(), ws1, ws3, ws2)
        I, H = cfg.I, cfg.H
        self.shared_w13 = self.w13[self.E_r * 2 * I:(self.E_r + 1) * 2 * I]
        self.shared_w2 = self.w2[self.E_r * H:(self.E_r + 1) * H]
        self.router_packed = moe.pack_router(cfg, w_router)
        self.bias = bias
        self.ws = moe.workspace(cfg, device=dev)
        T, K, E = cfg.T, cfg.K, cfg.E
        self.idx = torch.empty((T, K), dtype=torch.int32, device=dev)
        self.gate = torch.empty((T, K), dtype=torch.float32, device=dev)
        self.margin = torch.empty((T,), dtype=torch.float32, device=dev)
        self.counts = torch.empty((E + 1,), dtype=torch.int32, device=dev)
        self.offsets = torch.empty((E + 2,), dtype=torch.int32, device=dev)
        self.sorted = torch.empty((cfg.rows,), dtype=torch.int32, device=dev)
        self.y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        # owner side
        self.max_rows = int(max_rows)
        self.owner_ws = moe.workspace(self.owner_cfg(self.max_rows), device=dev)
        self.recv_gate = torch.empty((self.max_rows,), dtype=torch.float32, device=dev)
        self.recv_src = torch.empty((self.max_rows, 2), dtype=torch.int32, device=dev)
        self.recv_sorted = torch.empty((self.max_rows,), dtype=torch.int32, device=dev)
        self.recv_offsets = torch.empty((self.E_r + 2,), dtype=torch.int32, device=dev)
        self.dst_row = torch.empty((E,), dtype=torch.int32, device=dev)

    def owner_cfg(self, rows: int) -> moe.Config:
        return moe.Config(rows, self.cfg.H, self.cfg.I, self.E_r, 1, self.cfg.routed_scale, False)

    def recv_x_ptr(self, rows: int) -> int:
        return self.owner_ws.data_ptr() + workspace_offset(self.owner_cfg(rows), WS_TOKEN_ROWS)

    def slot_outputs_ptr(self) -> int:
        return self.ws.data_ptr() + workspace_offset(self.cfg, WS_SLOT_OUTPUTS)

    def route_and_permute(self, x, stream=None):
        moe.route_packed(self.cfg, x, self.router_packed, self.bias, self.ws,
                         out=(self.idx, self.gate, self.margin), stream=stream)
        moe.permute(self.cfg, self.idx, self.ws, out=(self.counts, self.offsets, self.sorted), stream=stream)

    def owner_forward(self, rows: int, stream=None):
        """The grouped GEMMs on the `rows` received rows (owner cfg: T = rows,
        K = 1, this rank's experts, no shared group; gates as received)."""
        oc = self.owner_cfg(rows)
        wts = (self.w13, self.w2)
        moe.expert_up(oc, wts, self.recv_offsets, self.recv_sorted, self.owner_ws, stream=stream)
        moe.expert_down(oc, wts, self.recv_gate, self.recv_offsets, self.recv_sorted, self.owner_ws,
                        stream=stream)


def virtual_forward(ranks: list[EpRank], xs: list[torch.Tensor], stream=None):
    """One expert-parallel step of R ranks emulated on one GPU: every rank's
    buffers are local, so the dispatch's and the return's "peer" stores are
    ordinary stores, and the steps of all ranks run in order on one stream (no
    kernel waits on another).  Returns each rank's y."""
    R = len(ranks)
    first = ranks[0].first
    for r, x in zip(ranks, xs):
        r.route_and_permute(x, stream)
    counts_all = torch.stack([r.counts[: r.cfg.E] for r in ranks])  # stands in for the all-gather
    for r in ranks:
        plan(r.cfg, first, r.rank, counts_all, r.dst_row, r.recv_offsets, r.recv_sorted, r.ws, stream)
    totals = [int(v) for v in counts_all.sum(dim=0).cpu().numpy()]  # the host needs the row counts
    rows = [sum(totals[first[o]:first[o + 1]]) for o in range(R)]
    recv_x = [ranks[o].recv_x_ptr(rows[o]) for o in range(R)]
    recv_gate = [ranks[o].recv_gate.data_ptr() for o in range(R)]
    recv_src = [ranks[o].recv_src.data_ptr() for o in range(R)]
    capacity = [min(ranks[o].max_rows, rows[o]) for o in range(R)]
    for r, x in zip(ranks, xs):
        dispatch(r.cfg, first, r.rank, r.dst_row, x, r.gate, r.offsets, r.sorted, recv_x, recv_gate, recv_src,
                 capacity, r.ws, stream)
    dst_y = [r.slot_outputs_ptr() for r in ranks]
    dst_rows = [r.cfg.T * r.cfg.K for r in ranks]
    for o in range(R):
        ranks[o].owner_forward(rows[o], stream)
        ret(ranks[o].owner_cfg(rows[o]), R, ranks[o].recv_src, dst_y, dst_rows, ranks[o].owner_ws, stream)
    for r, x in zip(ranks, xs):
        shared(r.cfg, r.shared_w13, r.shared_w2, x, r.ws, stream)
        moe.combine(r.cfg, r.ws, r.y, stream=stream)
    return [r.y for r in ranks]
