"""ctypes loader for librsm.so (the C ABI of include/rsm.h).

There is no fallback: if the in-tree library is missing or cannot be loaded, importing the
binding raises, so nothing can silently run another implementation.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "librsm.so")

RSM_OK, RSM_ERR_INVALID_ARG, RSM_ERR_UNSUPPORTED, RSM_ERR_CUDA, RSM_ERR_NONFINITE, \
    RSM_ERR_WORKSPACE, RSM_ERR_TIMEOUT = range(7)
RSM_F32, RSM_BF16 = 0, 1
RSM_DECAY_HEAD, RSM_DECAY_SLOT = 0, 1
RSM_PATH_AUTO, RSM_PATH_SIMT, RSM_PATH_TENSOR = 0, 1, 2
RSM_ROUTER_SIGMOID, RSM_ROUTER_SOFTMAX, RSM_ROUTER_SIGMOID_NORM, RSM_ROUTER_SOFTMAX_NORM = 0, 1, 2, 3
ROUTERS = {"sigmoid": RSM_ROUTER_SIGMOID, "softmax": RSM_ROUTER_SOFTMAX,
           "sigmoid_norm": RSM_ROUTER_SIGMOID_NORM, "softmax_norm": RSM_ROUTER_SOFTMAX_NORM}
RSM_FLAG_VALIDATE = 1
RSM_FLAG_TEST_STALL_ROUTING = 256

# Every symbol include/rsm.h declares (the CPU tests check the library exports all of them).
EXPORTED = ("rsm_route", "rsm_route_ex", "rsm_forward_workspace_size", "rsm_forward", "rsm_forward_selected_path",
            "rsm_forward_kernel_launches", "rsm_forward_set_profile_events",
            "rsm_decode_step", "rsm_backward_workspace_size", "rsm_backward",
            "rsm_status_string", "rsm_last_error", "rsm_get_device_status", "rsm_version",
            "rsm_forward_noalloc", "rsm_forward_noalloc_max_scratch")

_vp = ctypes.c_void_p
_int = ctypes.c_int


class ForwardArgs(ctypes.Structure):
    _fields_ = [("B", _int), ("T", _int), ("H", _int), ("M", _int), ("K", _int), ("Dv", _int),
                ("qkv_dtype", _int), ("decay", _int),
                ("q", _vp), ("k", _vp), ("v", _vp), ("logits", _vp), ("f", _vp), ("H0", _vp),
                ("o", _vp), ("HT", _vp), ("idx_out", _vp), ("score_out", _vp),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
                ("path", _int), ("flags", _int), ("router", _int), ("slot_counts", _vp)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("B", _int), ("H", _int), ("M", _int), ("K", _int), ("Dv", _int),
                ("qkv_dtype", _int), ("decay", _int),
                ("q", _vp), ("k", _vp), ("v", _vp), ("logits", _vp), ("f", _vp),
                ("state", _vp), ("o", _vp), ("idx_out", _vp), ("score_out", _vp),
                ("flags", _int), ("router", _int), ("slot_counts", _vp)]


class BackwardArgs(ctypes.Structure):
    _fields_ = [("B", _int), ("T", _int), ("H", _int), ("M", _int), ("K", _int), ("Dv", _int),
                ("qkv_dtype", _int), ("decay", _int),
                ("q", _vp), ("k", _vp), ("v", _vp), ("logits", _vp), ("f", _vp), ("H0", _vp),
                ("dO", _vp), ("dHT", _vp),
                ("dq", _vp), ("dk", _vp), ("dv", _vp), ("dlogits", _vp), ("df", _vp), ("dH0", _vp),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
                ("router", _int), ("flags", _int)]


class RSMError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"{status_string(status)}: {detail}")


_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"librsm.so is not built ({LIB_PATH}); run __graft_entry__.build()")
        lib = ctypes.CDLL(LIB_PATH)
        lib.rsm_route.argtypes = [_vp, ctypes.c_int64, _int, _int, _vp, _vp, _vp]
        lib.rsm_route.restype = _int
        lib.rsm_route_ex.argtypes = [_vp, ctypes.c_int64, _int, _int, _int, _int, _vp, _vp, _vp]
        lib.rsm_route_ex.restype = _int
        lib.rsm_forward_workspace_size.argtypes = [ctypes.POINTER(ForwardArgs)]
        lib.rsm_forward_workspace_size.restype = ctypes.c_size_t
        lib.rsm_forward.argtypes = [ctypes.POINTER(ForwardArgs), _vp]
        lib.rsm_forward.restype = _int
        lib.rsm_forward_selected_path.argtypes = [ctypes.POINTER(ForwardArgs)]
        lib.rsm_forward_selected_path.restype = _int
        lib.rsm_forward_kernel_launches.argtypes = [ctypes.POINTER(ForwardArgs)]
        lib.rsm_forward_kernel_launches.restype = _int
        lib.rsm_forward_set_profile_events.argtypes = [ctypes.POINTER(_vp), _int]
        lib.rsm_forward_set_profile_events.restype = _int
        lib.rsm_forward_noalloc.argtypes = [ctypes.POINTER(ForwardArgs), _vp]
        lib.rsm_forward_noalloc.restype = _int
        lib.rsm_forward_noalloc_max_scratch.argtypes = []
        lib.rsm_forward_noalloc_max_scratch.restype = ctypes.c_size_t
        lib.rsm_backward_workspace_size.argtypes = [ctypes.POINTER(BackwardArgs)]
        lib.rsm_backward_workspace_size.restype = ctypes.c_size_t
        lib.rsm_backward.argtypes = [ctypes.POINTER(BackwardArgs), _vp]
        lib.rsm_backward.restype = _int
        lib.rsm_decode_step.argtypes = [ctypes.POINTER(DecodeArgs), _vp]
        lib.rsm_decode_step.restype = _int
        lib.rsm_status_string.argtypes = [_int]
        lib.rsm_status_string.restype = ctypes.c_char_p
        lib.rsm_last_error.argtypes = []
        lib.rsm_last_error.restype = ctypes.c_char_p
        lib.rsm_get_device_status.argtypes = [_vp]
        lib.rsm_get_device_status.restype = _int
        lib.rsm_version.argtypes = []
        lib.rsm_version.restype = _int
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().rsm_status_string(status).decode()


def last_error() -> str:
    return load().rsm_last_error().decode()


def check(status: int) -> None:
    if status != RSM_OK:
        raise RSMError(status, last_error())
