"""librsm: a B200 (sm_100a) implementation of Raven's routing-state-model (RSM) mixer.

The product is the C ABI in include/rsm.h (librsm.so, built in-tree from csrc/). This package adds
a thin ctypes binding with the same three calls:

    route(logits, K)                          -> TopK slot indices and sigmoid scores
    forward(q, k, v, logits, f, K, H0=None)   -> chunked prefill: o and the final state H_T
    decode_step(q, k, v, logits, f, K, state) -> one generation token, state updated in place
    backward(q, k, v, logits, f, K, dO, dHT)  -> gradients of the prefill (RSMFunction: autograd)
"""
from .api import RSMFunction, backward, decode_step, device_status, forward, route  # noqa: F401
from ._lib import RSMError  # noqa: F401

__all__ = ["route", "forward", "backward", "decode_step", "device_status", "RSMFunction", "RSMError"]
