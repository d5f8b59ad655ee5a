"""rsm_forward_noalloc: the prefill for callers that cannot allocate device memory.

Such callers (work being recorded into a CUDA graph capture, programs whose allocator owns all
device memory, runtimes with a fixed memory plan) cannot hand rsm_forward the workspace it needs
when it splits a long sequence into segments. rsm_forward_noalloc uses a scratch array built into
the library instead. This file checks, through the C ABI, that two calls in a row give the same
results as rsm_forward with a caller-allocated workspace. It is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

TOL = 2e-2  # the tensor-core path's bar (bf16 q/k/v, fp32 state and accumulation)


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    from sparse_routed_slot_b200 import _lib
    return _lib


def _rel(x, ref):
    x = x.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    return float(np.max(np.abs(x - ref)) / max(np.sqrt(np.mean(ref ** 2)), 1e-300))


def _args(lib, x, K, o, HT):
    from sparse_routed_slot_b200 import api
    return api._forward_args(x["q"], x["k"], x["v"], x["logits"], x["f"], K, x["H0"], o, HT, None, None,
                             "auto", False)


def test_noalloc_matches_forward_on_two_calls_in_a_row(lib):
    from sparse_routed_slot_b200.workloads import make_inputs
    L = lib.load()
    assert L.rsm_forward_noalloc_max_scratch() == 16 << 20
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    B, H, M, K, Dv = 1, 2, 128, 16, 128
    for call, (T, decay, seed) in enumerate([(1000, "head", 11), (1537, "slot", 12)]):
        x = make_inputs(B, T, H, M, Dv, torch.bfloat16, decay, seed=seed, device="cuda", h0=True)
        # reference: the existing entry point with a workspace the caller allocates
        o_ref = torch.empty(B, T, H, Dv, device="cuda")
        h_ref = torch.empty(B, H, M, Dv, device="cuda")
        a = _args(lib, x, K, o_ref, h_ref)
        need = L.rsm_forward_workspace_size(ctypes.byref(a))
        assert 0 < need <= L.rsm_forward_noalloc_max_scratch()   # this case uses the scratch
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        a.workspace, a.workspace_bytes = ws.data_ptr(), need
        lib.check(L.rsm_forward(ctypes.byref(a), stream))
        # the allocation-free entry point: no workspace passed
        o = torch.full((B, T, H, Dv), float("nan"), device="cuda")
        h = torch.full((B, H, M, Dv), float("nan"), device="cuda")
        b = _args(lib, x, K, o, h)
        lib.check(L.rsm_forward_noalloc(ctypes.byref(b), stream))
        torch.cuda.synchronize()
        eo, eh = _rel(o, o_ref), _rel(h, h_ref)
        print(f"call {call}: o {eo:.2e}  H_T {eh:.2e}")
        assert eo <= TOL and eh <= TOL
