"""CPU oracle for the sigmoid-routed mixture-of-experts FFN (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this module.  The product path (the CUDA library and its binding)
never imports, links or calls it, and the two share no code.

The arithmetic lives in ``moe_oracle.c`` (plain C, double precision, OpenMP over
tokens).  This file only compiles it, marshals NumPy arrays into it and returns
NumPy arrays.  The definition it follows is the "Mixture of experts" step list of
the "GLM-5 . MoE transformer block" page (section "All 43 steps"), with the
selection-bias and renormalisation rules of the nnterp GLM-4.7-Flash / GLM-5
pages (note "The mixture: sigmoid scores, a selection bias, renormalized
weights").  Every function below names the equation it computes.

The second part, ``dsa_oracle.c``, states the sparse attention's key selection:
the indexer score of the same page's "All 43 steps" (S_I = sum_h w ReLU(q.k) /
(sqrt(32) sqrt(128)), causal mask) and the top-k key selection of the nnterp
glm_moe_dsa page ("Up to 2048 tokens the sparse attention is plain causal
attention"), pinned in ``tests/test_dsa_oracle_pins.py``.

Parity status: every function here is pinned by the not-gpu tests in
``tests/test_oracle_pins.py`` (closed forms, brute force, invariants, the
page's parameter count and a hand-derived worked example); none is "parity
unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRCS = [os.path.join(_HERE, "moe_oracle.c"), os.path.join(_HERE, "dsa_oracle.c")]
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_i64 = ctypes.c_int64
_int = ctypes.c_int
_dbl = ctypes.c_double
_vp = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile moe_oracle.c and dsa_oracle.c into liboracle.so next to them (gcc, OpenMP)."""
    stale = not os.path.exists(_LIB_PATH) or any(
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(src) for src in _SRCS)
    if force or stale:
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-o", tmp] + _SRCS + ["-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_param_count.restype = _i64
        lib.oracle_param_count.argtypes = [_i64, _i64, _i64, _i64]
        lib.oracle_rmsnorm.restype = _int
        lib.oracle_rmsnorm.argtypes = [_i64, _i64, _vp, _vp, _dbl, _vp]
        lib.oracle_logits.restype = _int
        lib.oracle_logits.argtypes = [_i64, _i64, _i64, _vp, _vp, _vp]
        lib.oracle_select.restype = _int
        lib.oracle_select.argtypes = [_i64, _i64, _i64, _dbl, _vp, _vp, _vp, _vp, _vp]
        lib.oracle_gates_for.restype = _int
        lib.oracle_gates_for.argtypes = [_i64, _i64, _i64, _dbl, _vp, _vp, _vp]
        lib.oracle_permute.restype = _int
        lib.oracle_permute.argtypes = [_i64, _i64, _i64, _int, _vp, _vp, _vp, _vp]
        lib.oracle_forward.restype = _int
        lib.oracle_forward.argtypes = [_i64, _i64, _i64, _i64, _i64, _int, _vp, _vp, _vp, _vp,
                                       _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp]
        lib.oracle_dsa_scores.restype = _int
        lib.oracle_dsa_scores.argtypes = [_i64, _i64, _i64, _i64, _i64, _vp, _vp, _vp, _vp]
        lib.oracle_dsa_select.restype = _int
        lib.oracle_dsa_select.argtypes = [_i64, _i64, _i64, _vp, _vp, _vp, _vp]
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(_vp)


def _check(rc, what):
    if rc != 0:
        raise ValueError("oracle %s failed with code %d" % (what, rc))


def _bf16(a):
    """bf16 data is passed around as uint16 bit patterns."""
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 arrays must be given as uint16 bit patterns, got %s" % a.dtype)
    return a


def param_count(H: int, I: int, E: int, n_shared: int = 1) -> int:
    """Parameters of one MoE block: router E*H, bias E, (E+n_shared) experts of 3*H*I."""
    return int(_load().oracle_param_count(H, I, E, n_shared))


def rmsnorm(x, gamma, eps: float):
    """x_ffn = x * gamma / sqrt(mean(x^2) + eps) per row, in double (x, gamma bf16 bits)."""
    x = _bf16(x)
    gamma = _bf16(gamma)
    T, H = x.shape
    assert gamma.shape == (H,)
    out = np.empty((T, H), dtype=np.float64)
    _check(_load().oracle_rmsnorm(T, H, _p(x), _p(gamma), float(eps), _p(out)), "rmsnorm")
    return out


def logits(x, w_r):
    """z = x W_r^T in double (equation z = x_ffn W_r; W_r stored [E, H])."""
    x = _bf16(x)
    w_r = np.ascontiguousarray(w_r, dtype=np.float32)
    T, H = x.shape
    E = w_r.shape[0]
    assert w_r.shape == (E, H)
    z = np.empty((T, E), dtype=np.float64)
    _check(_load().oracle_logits(T, H, E, _p(x), _p(w_r), _p(z)), "logits")
    return z


def select(z, bias, K: int, scale: float):
    """s = sigmoid(z); top-K of s + b (ties -> lower index); G = scale*s_sel/sum(s_sel).

    Returns (idx int32 [T,K], gate float64 [T,K], margin float64 [T])."""
    z = np.ascontiguousarray(z, dtype=np.float64)
    bias = np.ascontiguousarray(bias, dtype=np.float32)
    T, E = z.shape
    idx = np.empty((T, K), dtype=np.int32)
    gate = np.empty((T, K), dtype=np.float64)
    margin = np.empty((T,), dtype=np.float64)
    _check(_load().oracle_select(T, E, K, float(scale), _p(z), _p(bias), _p(idx), _p(gate),
                                 _p(margin)), "select")
    return idx, gate, margin


def route(x, w_r, bias, K: int, scale: float):
    """Router: logits then selection.  Returns (idx, gate, margin, z)."""
    z = logits(x, w_r)
    idx, gate, margin = select(z, bias, K, scale)
    return idx, gate, margin, z


def gates_for(z, idx, scale: float):
    """Gates of a given selection: G = scale * s_idx / sum over the slots of s_idx."""
    z = np.ascontiguousarray(z, dtype=np.float64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, E = z.shape
    K = idx.shape[1]
    gate = np.empty((T, K), dtype=np.float64)
    _check(_load().oracle_gates_for(T, E, K, float(scale), _p(z), _p(idx), _p(gate)), "gates_for")
    return gate


def permute(idx, E: int, has_shared: bool = True):
    """Counting sort of the assignments into expert groups (shared expert = group E).

    Returns (counts int32 [E+1], offsets int32 [E+2], sorted int32 [T*K (+T)])."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, K = idx.shape
    counts = np.empty((E + 1,), dtype=np.int32)
    offsets = np.empty((E + 2,), dtype=np.int32)
    sorted_ = np.empty((T * K + (T if has_shared else 0),), dtype=np.int32)
    _check(_load().oracle_permute(T, E, K, int(bool(has_shared)), _p(idx), _p(counts), _p(offsets),
                                  _p(sorted_)), "permute")
    return counts, offsets, sorted_


def forward(x, w1, w3, w2, ws1, ws3, ws2, idx, gate, tokens=None, has_shared=True,
            want_parts=False):
    """MoE output in double for the listed tokens (all when ``tokens`` is None).

    w1, w3: per-expert [I, H] bf16 (a 3-D array [E, I, H] or a list with None for
    experts no listed token uses); w2: per-expert [H, I].  Gates are used as given.
    Returns y [n, H]; with ``want_parts`` also (y_routed, y_shared, y_slot [n, K, H])."""
    x = _bf16(x)
    T, H = x.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    gate = np.ascontiguousarray(gate, dtype=np.float64)
    K = idx.shape[1]
    E = len(w1)
    keep = []

    def table(ws):
        arr = (_vp * E)()
        for e in range(E):
            if ws[e] is not None:
                a = _bf16(ws[e])
                keep.append(a)
                arr[e] = a.ctypes.data
        return arr

    t1, t3, t2 = table(w1), table(w3), table(w2)
    present = [np.asarray(w) for w in w1 if w is not None]
    if present:
        I = present[0].shape[0]
    elif has_shared:
        I = np.asarray(ws1).shape[0]
    else:
        I = 1
    if has_shared:
        ws1, ws3, ws2 = _bf16(ws1), _bf16(ws3), _bf16(ws2)
    else:
        ws1 = ws3 = ws2 = None
    if tokens is None:
        tok = None
        n = T
    else:
        tok = np.ascontiguousarray(tokens, dtype=np.int64)
        n = tok.shape[0]
    y = np.empty((n, H), dtype=np.float64)
    yr = np.empty((n, H), dtype=np.float64) if want_parts else None
    ys = np.empty((n, H), dtype=np.float64) if want_parts else None
    yk = np.empty((n, K, H), dtype=np.float64) if want_parts else None
    _check(_load().oracle_forward(T, H, I, E, K, int(bool(has_shared)), _p(x), t1, t3, t2,
                                  _p(ws1), _p(ws3), _p(ws2), _p(idx), _p(gate), n, _p(tok),
                                  _p(y), _p(yr), _p(ys), _p(yk)), "forward")
    if want_parts:
        return y, yr, ys, yk
    return y


# ---------------------------------------------------------------- sparse-attention key selection
# dsa_oracle.c: the indexer score of the "GLM-5 . MoE transformer block" page
# (section "All 43 steps") and the top-k key selection of the nnterp glm_moe_dsa
# page (section "Up to 2048 tokens the sparse attention is plain causal attention").

def dsa_scores(q, k, w):
    """Indexer scores in double: S[b,t,s] = sum_h w[b,t,h] ReLU(q[b,t,h].k[b,s]) / sqrt(NH*D)
    for s <= S-T+t, -inf for the keys the causal mask hides.

    q bf16 bits [B,T,NH,D], k bf16 bits [B,S,D], w float32 [B,T,NH] -> float64 [B,T,S]."""
    q = _bf16(q)
    k = _bf16(k)
    w = np.ascontiguousarray(w, dtype=np.float32)
    B, T, NH, D = q.shape
    S = k.shape[1]
    assert k.shape == (B, S, D) and w.shape == (B, T, NH)
    out = np.empty((B, T, S), dtype=np.float64)
    _check(_load().oracle_dsa_scores(B, T, S, NH, D, _p(q), _p(k), _p(w), _p(out)), "dsa_scores")
    return out


def dsa_select(scores, topk: int):
    """The first min(topk, S) keys of each row in (score descending, index ascending)
    order, listed in ascending key index.

    scores float64 [..., S] -> (sel int32 [..., n_sel], kth float64 [...], next float64 [...]):
    kth is the last taken key's score, next the first left out (-inf when all are taken)."""
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    lead = scores.shape[:-1]
    S = scores.shape[-1]
    R = int(np.prod(lead)) if lead else 1
    n_sel = min(int(topk), S)
    sel = np.empty((R, n_sel), dtype=np.int32)
    kth = np.empty((R,), dtype=np.float64)
    nxt = np.empty((R,), dtype=np.float64)
    _check(_load().oracle_dsa_select(R, S, int(topk), _p(scores), _p(sel), _p(kth), _p(nxt)),
           "dsa_select")
    return sel.reshape(lead + (n_sel,)), kth.reshape(lead), nxt.reshape(lead)
