"""Python binding of librsm: the same three calls as include/rsm.h, on torch CUDA tensors.

This layer only marshals arguments (shape/dtype checks, output allocation through torch,
pointers and the current CUDA stream). Every step of the mixer runs in the library's kernels.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib

_DTYPES = {torch.float32: _lib.RSM_F32, torch.bfloat16: _lib.RSM_BF16}
_PATHS = {"auto": _lib.RSM_PATH_AUTO, "simt": _lib.RSM_PATH_SIMT, "tensor": _lib.RSM_PATH_TENSOR}


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def route(logits: torch.Tensor, K: int, scores: bool = True, router: str = "sigmoid",
          validate: bool = False):
    """TopK routing of fp32 logits [..., M]. Returns (idx int32 [..., K], score fp32 [..., K]).
    router: "sigmoid" (default), "softmax", "sigmoid_norm" or "softmax_norm"."""
    _need(logits, "logits", torch.float32)
    M = logits.shape[-1]
    rows = logits.numel() // M if M else 0
    idx = torch.empty(*logits.shape[:-1], K, dtype=torch.int32, device=logits.device)
    sc = torch.empty(*logits.shape[:-1], K, dtype=torch.float32, device=logits.device) if scores else None
    L = _lib.load()
    if router == "sigmoid" and not validate:
        _lib.check(L.rsm_route(_ptr(logits), rows, M, K, _ptr(idx), _ptr(sc), _stream(logits.device)))
    else:
        _lib.check(L.rsm_route_ex(_ptr(logits), rows, M, K, _lib.ROUTERS[router],
                                  _lib.RSM_FLAG_VALIDATE if validate else 0, _ptr(idx), _ptr(sc),
                                  _stream(logits.device)))
    return idx, sc


def _forward_args(q, k, v, logits, f, K, H0, o, HT, idx, sc, path, validate, router="sigmoid",
                  counts=None) -> _lib.ForwardArgs:
    B, T, H, M = q.shape
    Dv = v.shape[-1]
    if q.dtype not in _DTYPES:
        raise ValueError("q, k, v must be float32 or bfloat16")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.dtype)
    _need(k, "k", shape=(B, T, H, M))
    _need(v, "v", shape=(B, T, H, Dv))
    _need(logits, "logits", torch.float32, (B, T, H, M))
    _need(f, "f", torch.float32)
    if tuple(f.shape) == (B, T, H):
        decay = _lib.RSM_DECAY_HEAD
    elif tuple(f.shape) == (B, T, H, M):
        decay = _lib.RSM_DECAY_SLOT
    else:
        raise ValueError(f"f must be [B,T,H] or [B,T,H,M], got {tuple(f.shape)}")
    if H0 is not None:
        _need(H0, "H0", torch.float32, (B, H, M, Dv))
    a = _lib.ForwardArgs()
    a.B, a.T, a.H, a.M, a.K, a.Dv = B, T, H, M, K, Dv
    a.qkv_dtype, a.decay = _DTYPES[q.dtype], decay
    a.q, a.k, a.v, a.logits, a.f = (t.data_ptr() for t in (q, k, v, logits, f))
    a.H0 = None if H0 is None else H0.data_ptr()
    a.o = o.data_ptr()
    a.HT = None if HT is None else HT.data_ptr()
    a.idx_out = None if idx is None else idx.data_ptr()
    a.score_out = None if sc is None else sc.data_ptr()
    a.path = _PATHS[path]
    a.flags = _lib.RSM_FLAG_VALIDATE if validate else 0
    a.router = _lib.ROUTERS[router]
    if counts is not None:
        _need(counts, "slot_counts", torch.int32, (B, H, M))
    a.slot_counts = None if counts is None else counts.data_ptr()
    return a


def workspace_bytes(args: _lib.ForwardArgs) -> int:
    n = _lib.load().rsm_forward_workspace_size(ctypes.byref(args))
    if n == ctypes.c_size_t(-1).value:
        _lib.check(_lib.load().rsm_forward(ctypes.byref(args), None))  # raises with the reason
    return n


def selected_path(args: _lib.ForwardArgs) -> str:
    """Which implementation rsm_forward runs for these arguments ("simt" or "tensor")."""
    p = _lib.load().rsm_forward_selected_path(ctypes.byref(args))
    if p < 0:
        _lib.check(_lib.load().rsm_forward(ctypes.byref(args), None))
    return "tensor" if p == _lib.RSM_PATH_TENSOR else "simt"


def kernel_launches(args: _lib.ForwardArgs) -> int:
    """Kernel launches one rsm_forward call makes for these arguments."""
    n = _lib.load().rsm_forward_kernel_launches(ctypes.byref(args))
    if n < 0:
        _lib.check(_lib.load().rsm_forward(ctypes.byref(args), None))
    return n


def forward(q, k, v, logits, f, K: int, H0=None, *, state: bool = True, routing: bool = False,
            path: str = "auto", validate: bool = False, out=None, workspace=None, router: str = "sigmoid",
            slot_counts=None):
    """Chunked prefill. q, k [B,T,H,M]; v [B,T,H,Dv]; logits [B,T,H,M] fp32; f [B,T,H] or
    [B,T,H,M] fp32; H0 [B,H,M,Dv] fp32 or None.

    Returns dict(o [B,T,H,Dv] fp32, HT [B,H,M,Dv] fp32 or None, idx, score [B,T,H,K] or None).
    `out` may supply preallocated tensors under the same keys; `workspace` a uint8 CUDA tensor.
    `router` picks the score variant; `slot_counts` (int32 [B,H,M]) gets the number of tokens
    that selected each slot added to it.
    """
    B, T, H, M = q.shape
    Dv = v.shape[-1]
    dev = q.device
    out = dict(out or {})
    o = out.get("o")
    if o is None:
        o = torch.empty(B, T, H, Dv, dtype=torch.float32, device=dev)
    HT = out.get("HT")
    if HT is None and state:
        HT = torch.empty(B, H, M, Dv, dtype=torch.float32, device=dev)
    idx = out.get("idx") if routing else None
    sc = out.get("score") if routing else None
    if routing:
        idx = idx if idx is not None else torch.empty(B, T, H, K, dtype=torch.int32, device=dev)
        sc = sc if sc is not None else torch.empty(B, T, H, K, dtype=torch.float32, device=dev)
    a = _forward_args(q, k, v, logits, f, K, H0, o, HT, idx, sc, path, validate, router, slot_counts)
    need = workspace_bytes(a)
    if need:
        if workspace is None or workspace.numel() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel()
    _lib.check(_lib.load().rsm_forward(ctypes.byref(a), _stream(dev)))
    return {"o": o, "HT": HT, "idx": idx, "score": sc}


def decode_step(q, k, v, logits, f, K: int, state, *, routing: bool = False, validate: bool = False,
                o=None, flags: int = 0, router: str = "sigmoid", slot_counts=None):
    """One token per (b,h). q, k [B,H,M]; v [B,H,Dv]; logits [B,H,M]; f [B,H] or [B,H,M];
    state [B,H,M,Dv] fp32 updated in place. Returns dict(o [B,H,Dv] fp32, idx, score).
    `flags` are extra RSM_FLAG_* bits passed through unchanged."""
    B, H, M = q.shape
    Dv = v.shape[-1]
    if q.dtype not in _DTYPES:
        raise ValueError("q, k, v must be float32 or bfloat16")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.dtype)
    _need(k, "k", shape=(B, H, M))
    _need(v, "v", shape=(B, H, Dv))
    _need(logits, "logits", torch.float32, (B, H, M))
    _need(f, "f", torch.float32)
    _need(state, "state", torch.float32, (B, H, M, Dv))
    if tuple(f.shape) == (B, H):
        decay = _lib.RSM_DECAY_HEAD
    elif tuple(f.shape) == (B, H, M):
        decay = _lib.RSM_DECAY_SLOT
    else:
        raise ValueError(f"f must be [B,H] or [B,H,M], got {tuple(f.shape)}")
    dev = q.device
    if o is None:
        o = torch.empty(B, H, Dv, dtype=torch.float32, device=dev)
    idx = torch.empty(B, H, K, dtype=torch.int32, device=dev) if routing else None
    sc = torch.empty(B, H, K, dtype=torch.float32, device=dev) if routing else None
    a = _lib.DecodeArgs()
    a.B, a.H, a.M, a.K, a.Dv = B, H, M, K, Dv
    a.qkv_dtype, a.decay = _DTYPES[q.dtype], decay
    a.q, a.k, a.v, a.logits, a.f = (t.data_ptr() for t in (q, k, v, logits, f))
    a.state, a.o = state.data_ptr(), o.data_ptr()
    a.idx_out = None if idx is None else idx.data_ptr()
    a.score_out = None if sc is None else sc.data_ptr()
    a.flags = (_lib.RSM_FLAG_VALIDATE if validate else 0) | flags
    a.router = _lib.ROUTERS[router]
    if slot_counts is not None:
        _need(slot_counts, "slot_counts", torch.int32, (B, H, M))
    a.slot_counts = None if slot_counts is None else slot_counts.data_ptr()
    _lib.check(_lib.load().rsm_decode_step(ctypes.byref(a), _stream(dev)))
    return {"o": o, "idx": idx, "score": sc}


def device_status(device=None) -> int:
    """Synchronizes the current stream and returns (and clears) the device status code."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return _lib.load().rsm_get_device_status(_stream(dev))


def backward(q, k, v, logits, f, K: int, dO=None, dHT=None, H0=None, *, validate: bool = False,
             out=None, workspace=None, flags: int = 0):
    """Gradients of rsm_forward (sigmoid router): q, k, v, logits, f, H0 as in forward();
    dO [B,T,H,Dv] fp32 and dHT [B,H,M,Dv] fp32 (None = zero). Returns dict(dq, dk, dlogits
    [B,T,H,M], dv [B,T,H,Dv], df (f's shape), dH0 [B,H,M,Dv]), all fp32. `flags` are extra
    RSM_FLAG_* bits passed through unchanged."""
    B, T, H, M = q.shape
    Dv = v.shape[-1]
    dev = q.device
    a0 = _forward_args(q, k, v, logits, f, K, H0, torch.empty(1, device=dev), None, None, None, "simt",
                       validate)  # shape and dtype checks shared with the forward
    a = _lib.BackwardArgs()
    for name in ("B", "T", "H", "M", "K", "Dv", "qkv_dtype", "decay", "q", "k", "v", "logits", "f", "H0",
                 "flags"):
        setattr(a, name, getattr(a0, name))
    if dO is not None:
        _need(dO, "dO", torch.float32, (B, T, H, Dv))
    if dHT is not None:
        _need(dHT, "dHT", torch.float32, (B, H, M, Dv))
    a.dO = None if dO is None else dO.data_ptr()
    a.dHT = None if dHT is None else dHT.data_ptr()
    out = dict(out or {})
    shapes = {"dq": (B, T, H, M), "dk": (B, T, H, M), "dlogits": (B, T, H, M), "dv": (B, T, H, Dv),
              "df": tuple(f.shape), "dH0": (B, H, M, Dv)}
    for name, shape in shapes.items():
        if out.get(name) is None:
            out[name] = torch.empty(shape, dtype=torch.float32, device=dev)
        _need(out[name], name, torch.float32, shape)
        setattr(a, name, out[name].data_ptr())
    a.router = _lib.RSM_ROUTER_SIGMOID
    a.flags = a.flags | flags
    L = _lib.load()
    need = L.rsm_backward_workspace_size(ctypes.byref(a))
    if need == ctypes.c_size_t(-1).value:
        _lib.check(L.rsm_backward(ctypes.byref(a), None))  # raises with the reason
    if need:
        if workspace is None or workspace.numel() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel()
    _lib.check(L.rsm_backward(ctypes.byref(a), _stream(dev)))
    return out


class RSMFunction(torch.autograd.Function):
    """The mixer as an autograd function: forward runs rsm_forward, backward runs rsm_backward.
    Inputs q, k, v, logits, f (and optionally H0); outputs o and H_T."""

    @staticmethod
    def forward(ctx, q, k, v, logits, f, K, H0=None):
        res = forward(q, k, v, logits, f, K, H0)
        ctx.K = K
        ctx.save_for_backward(q, k, v, logits, f, H0 if H0 is not None else torch.empty(0, device=q.device))
        ctx.has_h0 = H0 is not None
        return res["o"], res["HT"]

    @staticmethod
    def backward(ctx, dO, dHT):
        q, k, v, logits, f, H0 = ctx.saved_tensors
        g = backward(q, k, v, logits, f, ctx.K, None if dO is None else dO.float().contiguous(),
                     None if dHT is None else dHT.float().contiguous(), H0 if ctx.has_h0 else None)
        cast = lambda t, like: t.to(like.dtype)
        return (cast(g["dq"], q), cast(g["dk"], k), cast(g["dv"], v), g["dlogits"], g["df"], None,
                g["dH0"] if ctx.has_h0 else None)
