"""GPU parity of rsm_backward (gradients of the prefill) against the fp64 oracle's reverse sweep,
through the C ABI: dq, dk, dv, dlogits, df, dH0 at max|err| / rms(reference) <= 1e-4 (fp32
arithmetic), for both decay types, bf16 and fp32 inputs, ragged lengths and several shapes."""
import numpy as np
import pytest
import torch

from oracle import oracle
from sparse_routed_slot_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu

TOL = 1e-4


@pytest.fixture(scope="module")
def rsm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    import sparse_routed_slot_b200 as m
    return m


def rel(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(x - ref)) / max(np.sqrt(np.mean(ref ** 2)), 1e-300))


@pytest.mark.parametrize("M,K,Dv,T", [(32, 4, 32, 37), (64, 16, 64, 128), (128, 16, 128, 70), (256, 32, 64, 33)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("decay", ["head", "slot"])
def test_backward_matches_oracle(rsm, M, K, Dv, T, dtype, decay):
    B, H = 2, 2
    dev = torch.device("cuda")
    x = make_inputs(B, T, H, M, Dv, dtype, decay, seed=M + T, device=dev, h0=True)
    g = torch.Generator(device=dev).manual_seed(7)
    dO = torch.randn(B, T, H, Dv, generator=g, device=dev)
    dHT = torch.randn(B, H, M, Dv, generator=g, device=dev)
    out = rsm.backward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, dO, dHT, x["H0"])
    torch.cuda.synchronize()
    c = {n: t.float().cpu().numpy() for n, t in x.items()}
    r = oracle.backward(c["q"], c["k"], c["v"], c["logits"], c["f"], K, dO=dO.cpu().numpy(),
                        dHT=dHT.cpu().numpy(), H0=c["H0"])
    errs = {n: rel(out[n].cpu().numpy(), r[n]) for n in ("dq", "dk", "dv", "dlogits", "df", "dH0")}
    print(errs)
    assert all(e <= TOL for e in errs.values()), errs


@pytest.mark.parametrize("M,K,Dv,T", [(256, 32, 96, 21), (256, 256, 96, 9)])
def test_backward_large_state_layouts(rsm, M, K, Dv, T):
    """The largest states (M*Dv = 24576): the tape rows are read from global memory instead of
    travelling through the 8-slot ring (K = 32), and a 2-slot ring (K = M = 256)."""
    B, H = 1, 2
    dev = torch.device("cuda")
    x = make_inputs(B, T, H, M, Dv, torch.bfloat16, "slot", seed=M + K, device=dev, h0=True)
    g = torch.Generator(device=dev).manual_seed(11)
    dO = torch.randn(B, T, H, Dv, generator=g, device=dev)
    dHT = torch.randn(B, H, M, Dv, generator=g, device=dev)
    out = rsm.backward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, dO, dHT, x["H0"])
    torch.cuda.synchronize()
    c = {n: t.float().cpu().numpy() for n, t in x.items()}
    r = oracle.backward(c["q"], c["k"], c["v"], c["logits"], c["f"], K, dO=dO.cpu().numpy(),
                        dHT=dHT.cpu().numpy(), H0=c["H0"])
    errs = {n: rel(out[n].cpu().numpy(), r[n]) for n in ("dq", "dk", "dv", "dlogits", "df", "dH0")}
    assert all(e <= TOL for e in errs.values()), errs


def test_backward_without_output_gradient_and_zero_tokens(rsm):
    """dO = None (a loss on H_T only); and T = 0 (dH0 = dHT)."""
    B, T, H, M, K, Dv = 1, 50, 2, 64, 8, 64
    dev = torch.device("cuda")
    x = make_inputs(B, T, H, M, Dv, torch.float32, "head", seed=3, device=dev)
    dHT = torch.randn(B, H, M, Dv, generator=torch.Generator(device=dev).manual_seed(1), device=dev)
    out = rsm.backward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, None, dHT)
    torch.cuda.synchronize()
    c = {n: t.float().cpu().numpy() for n, t in x.items()}
    r = oracle.backward(c["q"], c["k"], c["v"], c["logits"], c["f"], K, dHT=dHT.cpu().numpy())
    assert np.all(out["dq"].cpu().numpy() == 0.0)
    for n in ("dk", "dv", "dlogits", "df", "dH0"):
        assert rel(out[n].cpu().numpy(), r[n]) <= TOL, n
    z = {n: t[:, :0].contiguous() for n, t in x.items()}
    out0 = rsm.backward(z["q"], z["k"], z["v"], z["logits"], z["f"], K, None, dHT)
    torch.cuda.synchronize()
    assert torch.equal(out0["dH0"], dHT)


def test_autograd_function_gradients(rsm):
    """RSMFunction: torch autograd through rsm_forward / rsm_backward gives the oracle's
    gradients of a scalar loss."""
    B, T, H, M, K, Dv = 1, 40, 2, 64, 8, 64
    dev = torch.device("cuda")
    x = make_inputs(B, T, H, M, Dv, torch.float32, "slot", seed=9, device=dev, h0=True)
    leaves = {n: t.clone().requires_grad_(True) for n, t in x.items()}
    o, HT = rsm.RSMFunction.apply(leaves["q"], leaves["k"], leaves["v"], leaves["logits"], leaves["f"], K,
                                  leaves["H0"])
    wo = torch.randn_like(o)
    loss = (o * wo).sum() + HT.square().sum()
    loss.backward()
    c = {n: t.float().cpu().numpy() for n, t in x.items()}
    fwd = oracle.forward(c["q"], c["k"], c["v"], c["logits"], c["f"], K, c["H0"])
    r = oracle.backward(c["q"], c["k"], c["v"], c["logits"], c["f"], K, dO=wo.cpu().numpy(),
                        dHT=2 * fwd["HT"], H0=c["H0"])
    for n, gname in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("logits", "dlogits"), ("f", "df"), ("H0", "dH0")):
        assert rel(leaves[n].grad.cpu().numpy(), r[gname]) <= 1e-3, n
