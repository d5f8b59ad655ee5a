"""GPU parity of the router variants and the per-slot selection counts, through the C ABI.

Router variants (the selected set is the same; only the score s in a = e^{s f} changes):
sigmoid (default), softmax over the row's M slots, and either one normalised over the K selected
slots. Selection counts: the number of tokens (prefill) or steps (decode) that selected each slot,
added to the caller's int32 [B,H,M] array. Bars as in test_gpu_parity: indices and counts
bit-exact, scores within 1e-6, o and the state at 1e-4 (fp32 arithmetic) or 2e-2 (tensor path).
"""
import numpy as np
import pytest
import torch

from oracle import oracle
from sparse_routed_slot_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu

ROUTERS = ["sigmoid", "softmax", "sigmoid_norm", "softmax_norm"]


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


@pytest.mark.parametrize("router", ROUTERS)
@pytest.mark.parametrize("M,K", [(32, 4), (128, 16), (256, 32)])
def test_route_variants(rsm, router, M, K):
    g = torch.Generator().manual_seed(M + K)
    lg = torch.cat([3 * torch.randn(300, M, generator=g), torch.round(2 * torch.randn(20, M, generator=g)) / 2])
    idx, sc = rsm.route(lg.cuda(), K, router=router)
    torch.cuda.synchronize()
    ri, rs = oracle.route(lg.numpy(), K, router)
    assert np.array_equal(idx.cpu().numpy(), ri)
    assert float(np.max(np.abs(sc.cpu().numpy() - rs))) <= 1e-6


@pytest.mark.parametrize("router", ROUTERS)
@pytest.mark.parametrize("path", ["simt", "tensor"])
@pytest.mark.parametrize("decay", ["head", "slot"])
def test_forward_variants_and_counts(rsm, router, path, decay):
    B, T, H, M, K, Dv = 2, 333, 3, 128, 16, 128
    x = make_inputs(B, T, H, M, Dv, torch.bfloat16, decay, seed=17, device="cuda", h0=True)
    counts = torch.full((B, H, M), 5, dtype=torch.int32, device="cuda")  # added to
    out = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, x["H0"], routing=True, path=path,
                      router=router, slot_counts=counts)
    torch.cuda.synchronize()
    c = {n: t.float().cpu().numpy() for n, t in x.items()}
    r = oracle.forward(c["q"], c["k"], c["v"], c["logits"], c["f"], K, c["H0"], router=router, want_counts=True)
    assert np.array_equal(out["idx"].cpu().numpy(), r["idx"])
    assert float(np.max(np.abs(out["score"].cpu().numpy() - r["score"]))) <= 1e-6
    assert np.array_equal(counts.cpu().numpy(), r["counts"] + 5)
    tol = 1e-4 if path == "simt" else 2e-2
    assert rel(out["o"].cpu().numpy(), r["o"]) <= tol
    assert rel(out["HT"].cpu().numpy(), r["HT"]) <= tol


def test_forward_counts_long_segmented(rsm):
    """A long stream split into segments (every segment's records counted once)."""
    B, T, H, M, K, Dv = 1, 5000, 2, 128, 16, 128
    x = make_inputs(B, T, H, M, Dv, torch.bfloat16, "head", seed=23, device="cuda")
    counts = torch.zeros((B, H, M), dtype=torch.int32, device="cuda")
    rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, slot_counts=counts)
    torch.cuda.synchronize()
    from oracle import brute
    lg = x["logits"].cpu().numpy()
    for h in range(H):
        assert np.array_equal(counts[0, h].cpu().numpy(), brute.selection_counts(lg[0, :, h], K))


@pytest.mark.parametrize("router", ROUTERS)
@pytest.mark.parametrize("M,Dv", [(64, 64), (128, 128)])
def test_decode_variants_and_counts(rsm, router, M, Dv):
    B, H, K, steps = 4, 5, 16, 4
    dev = torch.device("cuda")
    st = torch.randn(B, H, M, Dv, generator=torch.Generator(device=dev).manual_seed(3), device=dev)
    ref_state = st.double().cpu().numpy()
    counts = torch.zeros((B, H, M), dtype=torch.int32, device=dev)
    ref_counts = np.zeros((B, H, M), np.int64)
    for s in range(steps):
        x = make_inputs(B, 1, H, M, Dv, torch.bfloat16, "slot", seed=70 + s, device=dev)
        x = {n: t[:, 0].contiguous() for n, t in x.items()}
        d = rsm.decode_step(x["q"], x["k"], x["v"], x["logits"], x["f"], K, st, routing=True, router=router,
                            slot_counts=counts)
        torch.cuda.synchronize()
        xc = {n: t.float().cpu().numpy() for n, t in x.items()}
        r = oracle.decode_step(xc["q"], xc["k"], xc["v"], xc["logits"], xc["f"], K, ref_state, router=router)
        ref_state = r["state"]
        ref_counts += r["counts"]
        assert np.array_equal(d["idx"].cpu().numpy(), r["idx"])
        assert float(np.max(np.abs(d["score"].cpu().numpy() - r["score"]))) <= 1e-6
        assert rel(d["o"].cpu().numpy(), r["o"]) <= 1e-4
        assert rel(st.cpu().numpy(), ref_state) <= 1e-4
    assert np.array_equal(counts.cpu().numpy(), ref_counts)
