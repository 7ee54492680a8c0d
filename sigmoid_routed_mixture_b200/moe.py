"""Thin ctypes binding of libsrm_moe.so (declared in include/srm_moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  There is no
fallback of any kind: if the library is missing, every call raises.

    cfg = moe.Config(T, H, I, E, K, routed_scale=2.5)
    w13, w2 = moe.pack_weights(cfg, w1, w3, w2, ws1, ws3, ws2)
    ws = moe.workspace(cfg)
    idx, gate, margin = moe.route(cfg, x, w_router, bias, ws)
    counts, offsets, sorted_ = moe.permute(cfg, idx, ws)
    y = moe.forward(cfg, (w13, w2), x, gate, offsets, sorted_, ws)
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# SRM_MOE_LIBRARY may name another build of the library (e.g. for an A/B of two builds)
LIB_PATH = os.environ.get("SRM_MOE_LIBRARY") or os.path.join(_PKG, "libsrm_moe.so")

# Entry points declared in include/srm_moe.h.
SYMBOLS = (
    "moe_workspace_size",
    "moe_pack_weights",
    "moe_route",
    "moe_router_packed_size",
    "moe_pack_router",
    "moe_route_packed",
    "moe_permute",
    "moe_forward",
    "moe_gather_tokens",
    "moe_expert_up",
    "moe_expert_down",
    "moe_combine",
    "moe_combine_residual",
    "moe_rmsnorm",
    "moe_dense_mlp",
    "moe_get_device_error",
    "moe_status_string",
    "moe_permute_noalloc",
)

STATUS = {
    0: "MOE_OK",
    1: "MOE_ERR_ARG",
    2: "MOE_ERR_UNSUPPORTED",
    3: "MOE_ERR_ALIGN",
    4: "MOE_ERR_WORKSPACE",
    5: "MOE_ERR_BAD_INDEX",
    6: "MOE_ERR_TIMEOUT",
    7: "MOE_ERR_CUDA",
    8: "MOE_ERR_RANGE",
}


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__("%s: %s (%s)" % (what, STATUS.get(code, "?"), _status_string(code)))


class _Cfg(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("K", ctypes.c_int32), ("routed_scale", ctypes.c_float),
                ("has_shared", ctypes.c_int32)]


class _Weights(ctypes.Structure):
    _fields_ = [("w13", ctypes.c_void_p), ("w2", ctypes.c_void_p)]


@dataclasses.dataclass(frozen=True)
class Config:
    T: int
    H: int
    I: int
    E: int
    K: int
    routed_scale: float = 2.5
    has_shared: bool = True

    @classmethod
    def of(cls, w) -> "Config":
        """From a ``workloads.Workload``."""
        return cls(w.T, w.H, w.I, w.E, w.K, w.scale, w.has_shared)

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)

    def c(self) -> _Cfg:
        return _Cfg(self.T, self.H, self.I, self.E, self.K, self.routed_scale, int(bool(self.has_shared)))

    @classmethod
    def dense(cls, T: int, H: int, I: int) -> "Config":
        """A dense-MLP configuration (E = K = 0, the MLP in the shared-expert slot)."""
        return cls(T, H, I, 0, 0, 1.0, True)

    @property
    def rows(self) -> int:
        """Expert-sorted rows: T*K routed plus T shared."""
        return self.T * self.K + (self.T if self.has_shared else 0)


_lib = None


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libsrm_moe.so not found at %s; build it with "
                               "`python -m sigmoid_routed_mixture_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, P = ctypes.c_void_p, ctypes.POINTER
        L.moe_workspace_size.restype = ctypes.c_size_t
        L.moe_workspace_size.argtypes = [P(_Cfg)]
        L.moe_pack_weights.restype = ctypes.c_int
        L.moe_pack_weights.argtypes = [P(_Cfg)] + [vp] * 10
        L.moe_route.restype = ctypes.c_int
        L.moe_route.argtypes = [P(_Cfg)] + [vp] * 8 + [ctypes.c_size_t, vp]
        L.moe_router_packed_size.restype = ctypes.c_size_t
        L.moe_router_packed_size.argtypes = [P(_Cfg)]
        L.moe_pack_router.restype = ctypes.c_int
        L.moe_pack_router.argtypes = [P(_Cfg), vp, vp, vp]
        L.moe_route_packed.restype = ctypes.c_int
        L.moe_route_packed.argtypes = [P(_Cfg)] + [vp] * 8 + [ctypes.c_size_t, vp]
        L.moe_permute.restype = ctypes.c_int
        L.moe_permute.argtypes = [P(_Cfg), vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.moe_forward.restype = ctypes.c_int
        L.moe_forward.argtypes = [P(_Cfg), P(_Weights), vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.moe_gather_tokens.restype = ctypes.c_int
        L.moe_gather_tokens.argtypes = [P(_Cfg), vp, vp, vp, ctypes.c_size_t, vp]
        L.moe_expert_up.restype = ctypes.c_int
        L.moe_expert_up.argtypes = [P(_Cfg), P(_Weights), vp, vp, vp, ctypes.c_size_t, vp]
        L.moe_expert_down.restype = ctypes.c_int
        L.moe_expert_down.argtypes = [P(_Cfg), P(_Weights), vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.moe_combine.restype = ctypes.c_int
        L.moe_combine.argtypes = [P(_Cfg), vp, vp, ctypes.c_size_t, vp]
        L.moe_combine_residual.restype = ctypes.c_int
        L.moe_combine_residual.argtypes = [P(_Cfg), vp, vp, vp, ctypes.c_size_t, vp]
        L.moe_rmsnorm.restype = ctypes.c_int
        L.moe_rmsnorm.argtypes = [P(_Cfg), vp, vp, ctypes.c_float, vp, vp]
        L.moe_dense_mlp.restype = ctypes.c_int
        L.moe_dense_mlp.argtypes = [P(_Cfg), P(_Weights), vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.moe_get_device_error.restype = ctypes.c_int
        L.moe_get_device_error.argtypes = [vp, P(ctypes.c_int), vp]
        L.moe_permute_noalloc.restype = ctypes.c_int
        L.moe_permute_noalloc.argtypes = [P(_Cfg), vp, vp, vp, vp, vp]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_status_string.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def _status_string(code: int) -> str:
    try:
        return lib().moe_status_string(code).decode()
    except Exception:  # pragma: no cover - only when the library itself is missing
        return "?"


def _check(rc: int, what: str):
    if rc != 0:
        raise MoeError(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _req(t, dtype, shape, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.device.type != "cuda":
        raise ValueError("%s must be on a CUDA device" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t


def workspace_bytes(cfg: Config) -> int:
    n = lib().moe_workspace_size(ctypes.byref(cfg.c()))
    if n == 0:
        raise MoeError(1, "moe_workspace_size")
    return int(n)


def workspace(cfg: Config, device=None) -> torch.Tensor:
    """A workspace tensor (uint8) of moe_workspace_size bytes, its control words
    (the first 256 bytes: the device error word among them) zeroed."""
    ws = torch.empty(workspace_bytes(cfg), dtype=torch.uint8, device=device or "cuda")
    ws[:256].zero_()
    return ws


def pack_weights(cfg: Config, w1, w3, w2, ws1=None, ws3=None, ws2=None, stream=None, inexact=None):
    """Returns (w13 bf16 [(E+1)*2I, H], w2p fp16 [(E+1)*H, I]) in the kernels' layout.
    inexact: optional int32 [1] device tensor; receives the number of W2 values
    whose fp16 copy is not exact (saturated beyond 65504, or rounded below fp16's
    2^-24 spacing)."""
    E, I, H = cfg.E, cfg.I, cfg.H
    bf = torch.bfloat16
    if E > 0 or w1 is not None:
        _req(w1, bf, (E, I, H), "w1")
        _req(w3, bf, (E, I, H), "w3")
        _req(w2, bf, (E, H, I), "w2")
    if cfg.has_shared:
        _req(ws1, bf, (I, H), "ws1")
        _req(ws3, bf, (I, H), "ws3")
        _req(ws2, bf, (H, I), "ws2")
    dev = (w1 if w1 is not None else ws1).device
    w13 = torch.empty(((E + 1) * 2 * I, H), dtype=bf, device=dev)
    w2p = torch.empty(((E + 1) * H, I), dtype=torch.float16, device=dev)
    if inexact is not None:
        _req(inexact, torch.int32, (1,), "inexact")
    _check(lib().moe_pack_weights(ctypes.byref(cfg.c()), _ptr(w1), _ptr(w3), _ptr(w2), _ptr(ws1),
                                  _ptr(ws3), _ptr(ws2), _ptr(w13), _ptr(w2p), _ptr(inexact),
                                  _stream(stream)),
           "moe_pack_weights")
    return w13, w2p


def _route_outputs(cfg, x, want_margin, out):
    T, K = cfg.T, cfg.K
    if out is None:
        idx = torch.empty((T, K), dtype=torch.int32, device=x.device)
        gate = torch.empty((T, K), dtype=torch.float32, device=x.device)
        margin = torch.empty((T,), dtype=torch.float32, device=x.device) if want_margin else None
        return idx, gate, margin
    return out


def route(cfg: Config, x, w_router, bias, ws, want_margin=True, out=None, logits=None, stream=None):
    """Router: returns (topk_idx int32 [T,K], topk_gate fp32 [T,K], margin fp32 [T] or None).
    ``logits``: optional fp32 [T, E] tensor that receives z (router_logits)."""
    T, H, E = cfg.T, cfg.H, cfg.E
    _req(x, torch.bfloat16, (T, H), "x")
    _req(w_router, torch.float32, (E, H), "w_router")
    _req(bias, torch.float32, (E,), "bias")
    idx, gate, margin = _route_outputs(cfg, x, want_margin, out)
    _check(lib().moe_route(ctypes.byref(cfg.c()), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(idx),
                           _ptr(gate), _ptr(margin), _ptr(logits), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_route")
    return idx, gate, margin


def pack_router(cfg: Config, w_router, stream=None):
    """The exact three-part bf16 split of W_r (fp32 [E, H]) as a uint8 device
    tensor of moe_router_packed_size bytes, for route_packed."""
    _req(w_router, torch.float32, (cfg.E, cfg.H), "w_router")
    n = lib().moe_router_packed_size(ctypes.byref(cfg.c()))
    if n == 0:
        raise MoeError(1, "moe_router_packed_size")
    packed = torch.empty((n,), dtype=torch.uint8, device=w_router.device)
    _check(lib().moe_pack_router(ctypes.byref(cfg.c()), _ptr(w_router), _ptr(packed), _stream(stream)),
           "moe_pack_router")
    return packed


def route_packed(cfg: Config, x, w_router_packed, bias, ws, want_margin=True, out=None, logits=None,
                 stream=None):
    """route() with the router weights from pack_router: one kernel."""
    T, H, E = cfg.T, cfg.H, cfg.E
    _req(x, torch.bfloat16, (T, H), "x")
    n = lib().moe_router_packed_size(ctypes.byref(cfg.c()))
    _req(w_router_packed, torch.uint8, (n,), "w_router_packed")
    _req(bias, torch.float32, (E,), "bias")
    idx, gate, margin = _route_outputs(cfg, x, want_margin, out)
    _check(lib().moe_route_packed(ctypes.byref(cfg.c()), _ptr(x), _ptr(w_router_packed), _ptr(bias),
                                  _ptr(idx), _ptr(gate), _ptr(margin), _ptr(logits), _ptr(ws), ws.numel(),
                                  _stream(stream)),
           "moe_route_packed")
    return idx, gate, margin


def permute(cfg: Config, topk_idx, ws, out=None, stream=None):
    """Expert-sorted permutation: returns (counts [E+1], offsets [E+2], sorted [rows]) int32."""
    _req(topk_idx, torch.int32, (cfg.T, cfg.K), "topk_idx")
    dev = topk_idx.device
    if out is None:
        counts = torch.empty((cfg.E + 1,), dtype=torch.int32, device=dev)
        offsets = torch.empty((cfg.E + 2,), dtype=torch.int32, device=dev)
        sorted_ = torch.empty((cfg.rows,), dtype=torch.int32, device=dev)
    else:
        counts, offsets, sorted_ = out
    _check(lib().moe_permute(ctypes.byref(cfg.c()), _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                             _ptr(sorted_), _ptr(ws), ws.numel(), _stream(stream)), "moe_permute")
    return counts, offsets, sorted_


def permute_noalloc(cfg: Config, topk_idx, out=None, stream=None):
    """moe_permute without a workspace (library-held scratch; T*K <= 262144)."""
    _req(topk_idx, torch.int32, (cfg.T, cfg.K), "topk_idx")
    dev = topk_idx.device
    if out is None:
        counts = torch.empty((cfg.E + 1,), dtype=torch.int32, device=dev)
        offsets = torch.empty((cfg.E + 2,), dtype=torch.int32, device=dev)
        sorted_ = torch.empty((cfg.rows,), dtype=torch.int32, device=dev)
    else:
        counts, offsets, sorted_ = out
    _check(lib().moe_permute_noalloc(ctypes.byref(cfg.c()), _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                                     _ptr(sorted_), _stream(stream)), "moe_permute_noalloc")
    return counts, offsets, sorted_


def forward(cfg: Config, weights, x, topk_gate, offsets, sorted_, ws, y=None, stream=None):
    """Expert FFNs + combine; gates used as given.  Returns y bf16 [T, H]."""
    w13, w2p = weights
    _req(x, torch.bfloat16, (cfg.T, cfg.H), "x")
    _req(topk_gate, torch.float32, (cfg.T, cfg.K), "topk_gate")
    _req(offsets, torch.int32, (cfg.E + 2,), "offsets")
    _req(sorted_, torch.int32, (cfg.rows,), "sorted")
    _req(w13, torch.bfloat16, ((cfg.E + 1) * 2 * cfg.I, cfg.H), "w13")
    _req(w2p, torch.float16, ((cfg.E + 1) * cfg.H, cfg.I), "w2")
    if y is None:
        y = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=x.device)
    W = _Weights(w13.data_ptr(), w2p.data_ptr())
    _check(lib().moe_forward(ctypes.byref(cfg.c()), ctypes.byref(W), _ptr(x), _ptr(topk_gate),
                             _ptr(offsets), _ptr(sorted_), _ptr(y), _ptr(ws), ws.numel(),
                             _stream(stream)), "moe_forward")
    return y


def _weights_struct(cfg, weights):
    w13, w2p = weights
    _req(w13, torch.bfloat16, ((cfg.E + 1) * 2 * cfg.I, cfg.H), "w13")
    _req(w2p, torch.float16, ((cfg.E + 1) * cfg.H, cfg.I), "w2")
    return _Weights(w13.data_ptr(), w2p.data_ptr())


def gather_tokens(cfg: Config, x, sorted_, ws, stream=None):
    """Stage 1 of forward: token rows of x in expert-sorted order, into ws."""
    _req(x, torch.bfloat16, (cfg.T, cfg.H), "x")
    _check(lib().moe_gather_tokens(ctypes.byref(cfg.c()), _ptr(x), _ptr(sorted_), _ptr(ws), ws.numel(),
                                   _stream(stream)), "moe_gather_tokens")


def expert_up(cfg: Config, weights, offsets, sorted_, ws, stream=None):
    """Stage 2 of forward: h = silu(x W1) * (x W3) per expert-sorted row, into ws."""
    W_ = _weights_struct(cfg, weights)
    _check(lib().moe_expert_up(ctypes.byref(cfg.c()), ctypes.byref(W_), _ptr(offsets), _ptr(sorted_),
                               _ptr(ws), ws.numel(), _stream(stream)), "moe_expert_up")


def expert_down(cfg: Config, weights, topk_gate, offsets, sorted_, ws, stream=None):
    """Stage 3 of forward: gate * (h W2) per row, into its (token, slot) place in ws."""
    W_ = _weights_struct(cfg, weights)
    _check(lib().moe_expert_down(ctypes.byref(cfg.c()), ctypes.byref(W_), _ptr(topk_gate),
                                 _ptr(offsets), _ptr(sorted_), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_expert_down")


def combine(cfg: Config, ws, y, stream=None):
    """Stage 4 of forward: y = sum of slot outputs + shared output (bf16 [T, H])."""
    _check(lib().moe_combine(ctypes.byref(cfg.c()), _ptr(y), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_combine")
    return y


def combine_residual(cfg: Config, ws, residual, y, stream=None):
    """Stage 4 with the residual add: y = residual + slot outputs + shared output."""
    _req(residual, torch.bfloat16, (cfg.T, cfg.H), "residual")
    _check(lib().moe_combine_residual(ctypes.byref(cfg.c()), _ptr(residual), _ptr(y), _ptr(ws), ws.numel(),
                                      _stream(stream)), "moe_combine_residual")
    return y


def rmsnorm(cfg: Config, x, gamma, eps=1e-5, out=None, stream=None):
    """Pre-FFN RMSNorm: x * gamma / sqrt(mean(x^2) + eps) per row (bf16 in and out)."""
    _req(x, torch.bfloat16, (cfg.T, cfg.H), "x")
    _req(gamma, torch.bfloat16, (cfg.H,), "gamma")
    if out is None:
        out = torch.empty_like(x)
    _check(lib().moe_rmsnorm(ctypes.byref(cfg.c()), _ptr(x), _ptr(gamma), float(eps), _ptr(out),
                             _stream(stream)), "moe_rmsnorm")
    return out


def dense_mlp(cfg: Config, weights, x, ws, residual=None, y=None, stream=None):
    """Dense SwiGLU MLP (cfg from Config.dense): y = (residual +) W2 (silu(W1 x) * W3 x)."""
    _req(x, torch.bfloat16, (cfg.T, cfg.H), "x")
    if residual is not None:
        _req(residual, torch.bfloat16, (cfg.T, cfg.H), "residual")
    if y is None:
        y = torch.empty_like(x)
    W_ = _weights_struct(cfg, weights)
    _check(lib().moe_dense_mlp(ctypes.byref(cfg.c()), ctypes.byref(W_), _ptr(x), _ptr(residual), _ptr(y),
                               _ptr(ws), ws.numel(), _stream(stream)), "moe_dense_mlp")
    return y


def device_error(ws, stream=None) -> int:
    """Read and clear the workspace's device error word (synchronises the stream)."""
    st = ctypes.c_int(0)
    _check(lib().moe_get_device_error(_ptr(ws), ctypes.byref(st), _stream(stream)),
           "moe_get_device_error")
    return int(st.value)


class MoeBlock:
    """One MoE block with packed weights and a workspace: ``y = block(x)``."""

    def __init__(self, cfg: Config, w_router, bias, w1, w3, w2, ws1=None, ws3=None, ws2=None,
                 packed=None):
        self.cfg = cfg
        self.w_router = w_router
        self.bias = bias
        # packed: (w13, w2) from pack_weights for this block's H, I and E, shared
        # with another block of the same shapes instead of packing again
        self.weights = packed if packed is not None else pack_weights(cfg, w1, w3, w2, ws1, ws3, ws2)
        self.router_packed = pack_router(cfg, w_router)
        self.ws = workspace(cfg, device=w_router.device)
        dev = w_router.device
        T, K, E = cfg.T, cfg.K, cfg.E
        self.idx = torch.empty((T, K), dtype=torch.int32, device=dev)
        self.gate = torch.empty((T, K), dtype=torch.float32, device=dev)
        self.margin = torch.empty((T,), dtype=torch.float32, device=dev)
        self.counts = torch.empty((E + 1,), dtype=torch.int32, device=dev)
        self.offsets = torch.empty((E + 2,), dtype=torch.int32, device=dev)
        self.sorted = torch.empty((cfg.rows,), dtype=torch.int32, device=dev)
        self.y = torch.empty((T, cfg.H), dtype=torch.bfloat16, device=dev)

    def sublayer(self, x_resid, gamma, eps=1e-5, stream=None, logits=None):
        """The decoder block's FFN sublayer: x' + MoE(RMSNorm(x')) (bf16 [T, H])."""
        cfg = self.cfg
        x_ffn = rmsnorm(cfg, x_resid, gamma, eps, stream=stream)
        route_packed(cfg, x_ffn, self.router_packed, self.bias, self.ws,
                     out=(self.idx, self.gate, self.margin), logits=logits, stream=stream)
        permute(cfg, self.idx, self.ws, out=(self.counts, self.offsets, self.sorted), stream=stream)
        gather_tokens(cfg, x_ffn, self.sorted, self.ws, stream=stream)
        expert_up(cfg, self.weights, self.offsets, self.sorted, self.ws, stream=stream)
        expert_down(cfg, self.weights, self.gate, self.offsets, self.sorted, self.ws, stream=stream)
        combine_residual(cfg, self.ws, x_resid, self.y, stream=stream)
        return self.y, x_ffn

    def __call__(self, x, stream=None, logits=None):
        route_packed(self.cfg, x, self.router_packed, self.bias, self.ws,
                     out=(self.idx, self.gate, self.margin), logits=logits, stream=stream)
        permute(self.cfg, self.idx, self.ws, out=(self.counts, self.offsets, self.sorted), stream=stream)
        return forward(self.cfg, self.weights, x, self.gate, self.offsets, self.sorted, self.ws, y=self.y,
                       stream=stream)
