"""TEST INFRASTRUCTURE ONLY: ctypes front end of the fp64 C oracle (rsm_oracle.c).

Only tests/, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline leg may import this module.
The oracle is a plain sequential recurrence over tokens (see the header of rsm_oracle.c for what
it computes and which passages it follows). It shares nothing with the CUDA library: it is
compiled by gcc from its own single C file, and it receives plain numpy arrays.

Inputs are numpy float32 arrays holding exactly the values the device sees (bf16 tensors are
widened to float32 first, which is exact). State and outputs are float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rsm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liborsm_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile rsm_oracle.c into a shared library next to it (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def bind(lib):
    """Declares the C signatures on a loaded oracle library (also used for test mutants)."""
    f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
    vp = ctypes.c_void_p
    lib.rsmo_forward.argtypes = [ctypes.c_int] * 7 + [f32p] * 5 + [vp] * 5 + [ctypes.c_int]
    lib.rsmo_forward.restype = ctypes.c_int
    lib.rsmo_route.argtypes = [f32p, ctypes.c_longlong, ctypes.c_int, ctypes.c_int, vp, vp]
    lib.rsmo_route.restype = ctypes.c_int
    lib.rsmo_forward_ex.argtypes = [ctypes.c_int] * 7 + [f32p] * 5 + [vp] * 5 + [ctypes.c_int, vp, ctypes.c_int]
    lib.rsmo_forward_ex.restype = ctypes.c_int
    lib.rsmo_route_ex.argtypes = [f32p, ctypes.c_longlong, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp]
    lib.rsmo_route_ex.restype = ctypes.c_int
    if hasattr(lib, "rsmo_backward"):
        lib.rsmo_backward.argtypes = [ctypes.c_int] * 7 + [f32p] * 5 + [vp] * 9 + [ctypes.c_int]
        lib.rsmo_backward.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = bind(ctypes.CDLL(build()))
    return _lib


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# Router variants: the score of a selected slot is its sigmoid (default) or its softmax over all M
# slots of the row, optionally normalised over the K selected slots to sum to one.
ROUTERS = {"sigmoid": 0, "softmax": 1, "sigmoid_norm": 2, "softmax_norm": 3}


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def forward(q, k, v, logits, f, K: int, H0=None, want_idx: bool = True, nthreads: int | None = None,
            router: str = "sigmoid", want_counts: bool = False):
    """Sequential fp64 recurrence over all tokens.

    q, k, logits: [B,T,H,M]; v: [B,T,H,Dv]; f: [B,T,H] (per-head decay) or [B,T,H,M] (per-slot).
    H0: optional [B,H,M,Dv] (zeros when None). router: a key of ROUTERS. Returns dict(o, HT, idx,
    score, counts) with o [B,T,H,Dv] float64, HT [B,H,M,Dv] float64, idx [B,T,H,K] int32,
    score [B,T,H,K] float64, counts [B,H,M] int32 (tokens that selected each slot) or None.
    """
    q, k, v, logits, f = map(_f32, (q, k, v, logits, f))
    B, T, H, M = q.shape
    Dv = v.shape[-1]
    assert k.shape == q.shape and logits.shape == q.shape and v.shape == (B, T, H, Dv)
    if f.shape == (B, T, H):
        per_slot = 0
    elif f.shape == (B, T, H, M):
        per_slot = 1
    else:
        raise ValueError(f"bad f shape {f.shape}")
    h0 = None if H0 is None else np.ascontiguousarray(np.asarray(H0, dtype=np.float64))
    if h0 is not None:
        assert h0.shape == (B, H, M, Dv)
    o = np.zeros((B, T, H, Dv), np.float64)
    HT = np.zeros((B, H, M, Dv), np.float64)
    idx = np.zeros((B, T, H, K), np.int32) if want_idx else None
    score = np.zeros((B, T, H, K), np.float64) if want_idx else None
    counts = np.zeros((B, H, M), np.int32) if want_counts else None
    rc = _load().rsmo_forward_ex(B, T, H, M, K, Dv, per_slot, q, k, v, logits, f, _ptr(h0), _ptr(o),
                                 _ptr(HT), _ptr(idx), _ptr(score), ROUTERS[router], _ptr(counts),
                                 nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle rejected the sizes")
    return {"o": o, "HT": HT, "idx": idx, "score": score, "counts": counts}


def decode_step(q, k, v, logits, f, K: int, state, nthreads: int | None = None, router: str = "sigmoid"):
    """One generation step on a carried state (returns a new state; the argument is not changed).

    q, k, logits: [B,H,M]; v: [B,H,Dv]; f: [B,H] or [B,H,M]; state: [B,H,M,Dv].
    """
    q, k, v, logits, f = map(_f32, (q, k, v, logits, f))
    fx = f[:, None] if f.ndim in (2, 3) else f
    out = forward(q[:, None], k[:, None], v[:, None], logits[:, None], fx, K, H0=state,
                  nthreads=nthreads, router=router, want_counts=True)
    return {"o": out["o"][:, 0], "state": out["HT"], "idx": out["idx"][:, 0],
            "score": out["score"][:, 0], "counts": out["counts"]}


def route(logits, K: int, router: str = "sigmoid"):
    """TopK (rank order: logit desc, index asc) and fp64 scores of the router variant for rows
    [N, M]."""
    lg = _f32(logits)
    N, M = lg.shape
    idx = np.zeros((N, K), np.int32)
    score = np.zeros((N, K), np.float64)
    if _load().rsmo_route_ex(lg, N, M, K, ROUTERS[router], _ptr(idx), _ptr(score)) != 0:
        raise ValueError("oracle rejected the sizes")
    return idx, score


def backward(q, k, v, logits, f, K: int, dO=None, dHT=None, H0=None, nthreads: int | None = None):
    """Gradients of the recurrence (sigmoid router) for the loss whose gradients with respect to
    o and H_T are dO [B,T,H,Dv] and dHT [B,H,M,Dv] (None = 0). Returns dict(dq, dk, dlogits
    [B,T,H,M], dv [B,T,H,Dv], df (f's shape), dH0 [B,H,M,Dv]), all float64."""
    q, k, v, logits, f = map(_f32, (q, k, v, logits, f))
    B, T, H, M = q.shape
    Dv = v.shape[-1]
    per_slot = 1 if f.shape == (B, T, H, M) else 0
    if not per_slot and f.shape != (B, T, H):
        raise ValueError(f"bad f shape {f.shape}")
    def d64(x):
        return None if x is None else np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    h0, do, dht = d64(H0), d64(dO), d64(dHT)
    out = {"dq": np.zeros((B, T, H, M)), "dk": np.zeros((B, T, H, M)), "dlogits": np.zeros((B, T, H, M)),
           "dv": np.zeros((B, T, H, Dv)), "df": np.zeros(f.shape), "dH0": np.zeros((B, H, M, Dv))}
    rc = _load().rsmo_backward(B, T, H, M, K, Dv, per_slot, q, k, v, logits, f, _ptr(h0), _ptr(do), _ptr(dht),
                               _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dlogits"]),
                               _ptr(out["df"]), _ptr(out["dH0"]), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle rejected the sizes")
    return out
