"""rsm_forward_noalloc: the prefill for callers that cannot allocate device memory.

Such callers (work being recorded into a CUDA graph capture, programs whose allocator owns all
device memory, runtimes with a fixed memory plan) cannot hand rsm_forward the workspace its
tensor-core path needs (routing records, and segment states when a long sequence is split).
rsm_forward_noalloc uses a scratch array built into the library instead. Through the C ABI this
file checks that:
* two calls in a row give bit-identical results to rsm_forward with a caller-allocated workspace
  (the same kernels run on the same inputs; the second call finds the first call's leftovers in
  the shared array, and its result is also checked against the fp64 oracle);
* sizes whose scratch would exceed the array are refused before any launch, outputs untouched.
It is named to be collected last.
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
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(x - ref)) / max(np.sqrt(np.mean(ref ** 2)), 1e-300))


def _args(x, K, o, HT):
    from sparse_routed_slot_b200 import api
    return api._forward_args(x["q"], x["k"], x["v"], x["logits"], x["f"], K, x.get("H0"), o, HT, None, None,
                             "auto", False)


def test_noalloc_matches_forward_on_two_calls_in_a_row(lib):
    from oracle import oracle
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
        a = _args(x, K, o_ref, h_ref)
        need = L.rsm_forward_workspace_size(ctypes.byref(a))
        assert 0 < need <= L.rsm_forward_noalloc_max_scratch()   # this case uses the scratch
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        a.workspace, a.workspace_bytes = ws.data_ptr(), need
        lib.check(L.rsm_forward(ctypes.byref(a), stream))
        # the allocation-free entry point: no workspace passed
        o = torch.full((B, T, H, Dv), float("nan"), device="cuda")
        h = torch.full((B, H, M, Dv), float("nan"), device="cuda")
        b = _args(x, K, o, h)
        lib.check(L.rsm_forward_noalloc(ctypes.byref(b), stream))
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref), f"call {call}: o differs from rsm_forward"
        assert torch.equal(h, h_ref), f"call {call}: H_T differs from rsm_forward"
        if call == 1:
            c = {n: t.float().cpu().numpy() for n, t in x.items()}
            r = oracle.forward(c["q"], c["k"], c["v"], c["logits"], c["f"], K, c["H0"], want_idx=False)
            eo, eh = _rel(o.cpu().numpy(), r["o"]), _rel(h.cpu().numpy(), r["HT"])
            print(f"second call vs oracle: o {eo:.2e}  H_T {eh:.2e}")
            assert eo <= TOL and eh <= TOL


def test_noalloc_refuses_sizes_beyond_its_scratch(lib):
    """The long-context shape (B=1, T=32768, H=16) needs about 75 MB of routing records: refused
    with RSM_ERR_WORKSPACE before anything is launched, so the outputs keep their contents."""
    L = lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    B, T, H, M, K, Dv = 1, 32768, 16, 128, 16, 128
    x = {n: torch.zeros(B, T, H, M, dtype=torch.bfloat16, device="cuda") for n in ("q", "k")}
    x["v"] = torch.zeros(B, T, H, Dv, dtype=torch.bfloat16, device="cuda")
    x["logits"] = torch.zeros(B, T, H, M, device="cuda")
    x["f"] = torch.zeros(B, T, H, device="cuda")
    o = torch.full((B, T, H, Dv), float("nan"), device="cuda")
    h = torch.full((B, H, M, Dv), float("nan"), device="cuda")
    a = _args(x, K, o, h)
    assert L.rsm_forward_workspace_size(ctypes.byref(a)) > L.rsm_forward_noalloc_max_scratch()
    rc = L.rsm_forward_noalloc(ctypes.byref(a), stream)
    assert rc == lib.RSM_ERR_WORKSPACE
    assert "scratch" in lib.last_error()
    torch.cuda.synchronize()
    assert torch.isnan(o).all() and torch.isnan(h).all()
