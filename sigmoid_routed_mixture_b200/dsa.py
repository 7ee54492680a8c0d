"""Thin ctypes binding of the sparse-attention key selection in libsrm_moe.so
(declared in include/srm_dsa.h).

Argument marshalling only: the scores and the top-k run in the library's CUDA
kernels; PyTorch supplies device memory and the current stream.  No fallback:
if the library is missing, every call raises.

    cfg = dsa.Config(B, T, S)                 # GLM-5: 32 heads x 128, top 2048
    ws = dsa.workspace(cfg)
    sel = dsa.select(cfg, q, k, w, ws)        # int32 [B, T, min(topk, S)]
"""
from __future__ import annotations

import ctypes
import dataclasses

import torch

from . import moe

SYMBOLS = ("dsa_workspace_size", "dsa_scores", "dsa_topk", "dsa_select")


class _Cfg(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("T", ctypes.c_int32), ("S", ctypes.c_int32),
                ("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("topk", ctypes.c_int32)]


@dataclasses.dataclass(frozen=True)
class Config:
    B: int
    T: int
    S: int
    n_heads: int = 32
    head_dim: int = 128
    topk: int = 2048

    def c(self) -> _Cfg:
        return _Cfg(self.B, self.T, self.S, self.n_heads, self.head_dim, self.topk)

    @property
    def n_sel(self) -> int:
        return min(self.topk, self.S)


_bound = False


def lib():
    global _bound
    L = moe.lib()
    if not _bound:
        vp, P = ctypes.c_void_p, ctypes.POINTER
        L.dsa_workspace_size.restype = ctypes.c_size_t
        L.dsa_workspace_size.argtypes = [P(_Cfg)]
        L.dsa_scores.restype = ctypes.c_int
        L.dsa_scores.argtypes = [P(_Cfg), vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.dsa_topk.restype = ctypes.c_int
        L.dsa_topk.argtypes = [P(_Cfg), vp, vp, vp, ctypes.c_size_t, vp]
        L.dsa_select.restype = ctypes.c_int
        L.dsa_select.argtypes = [P(_Cfg), vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        _bound = True
    return L


def workspace_bytes(cfg: Config) -> int:
    n = lib().dsa_workspace_size(ctypes.byref(cfg.c()))
    if n == 0:
        raise moe.MoeError(2, "dsa_workspace_size")
    return int(n)


def workspace(cfg: Config, device=None) -> torch.Tensor:
    """A zeroed workspace tensor (uint8) of dsa_workspace_size bytes."""
    return torch.zeros(workspace_bytes(cfg), dtype=torch.uint8, device=device or "cuda")


def _inputs(cfg: Config, q, k, w):
    moe._req(q, torch.bfloat16, (cfg.B, cfg.T, cfg.n_heads, cfg.head_dim), "q")
    moe._req(k, torch.bfloat16, (cfg.B, cfg.S, cfg.head_dim), "k")
    moe._req(w, torch.float32, (cfg.B, cfg.T, cfg.n_heads), "w")


def scores(cfg: Config, q, k, w, ws, out=None, stream=None):
    """Indexer scores fp32 [B, T, S]; entries a query cannot see are left as they were
    (``out`` if given, else a tensor filled with -inf)."""
    _inputs(cfg, q, k, w)
    if out is None:
        out = torch.full((cfg.B, cfg.T, cfg.S), float("-inf"), dtype=torch.float32, device=q.device)
    moe._req(out, torch.float32, (cfg.B, cfg.T, cfg.S), "out")
    moe._check(lib().dsa_scores(ctypes.byref(cfg.c()), moe._ptr(q), moe._ptr(k), moe._ptr(w),
                                moe._ptr(out), moe._ptr(ws), ws.numel(), moe._stream(stream)),
               "dsa_scores")
    return out


def topk(cfg: Config, sc, ws, out=None, stream=None):
    """Top-k key indices int32 [B, T, min(topk, S)] (ascending) from scores."""
    moe._req(sc, torch.float32, (cfg.B, cfg.T, cfg.S), "scores")
    if out is None:
        out = torch.empty((cfg.B, cfg.T, cfg.n_sel), dtype=torch.int32, device=sc.device)
    moe._req(out, torch.int32, (cfg.B, cfg.T, cfg.n_sel), "out")
    moe._check(lib().dsa_topk(ctypes.byref(cfg.c()), moe._ptr(sc), moe._ptr(out), moe._ptr(ws),
                              ws.numel(), moe._stream(stream)), "dsa_topk")
    return out


def select(cfg: Config, q, k, w, ws, out=None, scores_out=None, stream=None):
    """Scores then top-k in one call; returns int32 [B, T, min(topk, S)]."""
    _inputs(cfg, q, k, w)
    if out is None:
        out = torch.empty((cfg.B, cfg.T, cfg.n_sel), dtype=torch.int32, device=q.device)
    moe._req(out, torch.int32, (cfg.B, cfg.T, cfg.n_sel), "out")
    if scores_out is not None:
        moe._req(scores_out, torch.float32, (cfg.B, cfg.T, cfg.S), "scores_out")
    moe._check(lib().dsa_select(ctypes.byref(cfg.c()), moe._ptr(q), moe._ptr(k), moe._ptr(w),
                                moe._ptr(out), moe._ptr(scores_out), moe._ptr(ws), ws.numel(),
                                moe._stream(stream)), "dsa_select")
    return out
