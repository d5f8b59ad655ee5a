"""GPU parity of the CUDA library against the fp64 CPU oracle, through the C ABI.

Bars (stated for this path): TopK indices bit-exact; router scores within 1e-6; o and H_T within
max|err| / rms(reference) <= 1e-4 for fp32 arithmetic (the CUDA-core path, any input dtype) and
<= 2e-2 for the tensor-core path with bf16 q/k/v and fp32 state and accumulation. Slots that are
not selected keep their bits.
"""
import numpy as np
import pytest
import torch

from oracle import oracle
from sparse_routed_slot_b200.workloads import WORKLOADS, make_inputs, make_workload_inputs

pytestmark = pytest.mark.gpu

TOL_FP32 = 1e-4
TOL_BF16 = 2e-2


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


def host(d):
    return {n: t.float().cpu().numpy() for n, t in d.items()}


def tol_for(path, dtype):
    return TOL_FP32 if (path == "simt" or dtype == torch.float32) else TOL_BF16


# ------------------------------------------------------------------------------------ routing


def _route_rows(M, n, seed):
    g = torch.Generator().manual_seed(seed)
    rows = [torch.randn(n, M, generator=g)]
    rows.append(torch.round(4 * torch.randn(n, M, generator=g)) / 4)           # many exact ties
    rows.append(torch.zeros(4, M))                                             # all equal
    z = torch.zeros(4, M)
    z[:, ::2] = -0.0
    rows.append(z)                                                             # signed zeros
    rows.append(20 + torch.randn(n, M, generator=g))                           # saturated sigmoid
    near = torch.full((n, M), 1.5)
    bump = torch.rand(n, M, generator=g) < 0.5
    near[bump] = torch.nextafter(torch.tensor(1.5), torch.tensor(2.0))
    rows.append(near)                                                          # one-ulp near ties
    return torch.cat(rows).float().contiguous()


@pytest.mark.parametrize("M", [32, 64, 128, 256])
@pytest.mark.parametrize("K", [1, 16, 32])
def test_route_bit_exact(rsm, M, K):
    if K > M:
        pytest.skip("K > M")
    rows = _route_rows(M, 512, seed=M * 7 + K)
    idx, sc = rsm.route(rows.cuda(), K)
    torch.cuda.synchronize()
    ri, rs = oracle.route(rows.numpy(), K)
    assert np.array_equal(idx.cpu().numpy(), ri)
    assert float(np.max(np.abs(sc.cpu().numpy() - rs))) <= 1e-6


def test_route_dense_and_empty(rsm):
    rows = _route_rows(64, 64, seed=5)
    idx, _ = rsm.route(rows.cuda(), 64)
    torch.cuda.synchronize()
    ri, _ = oracle.route(rows.numpy(), 64)
    assert np.array_equal(idx.cpu().numpy(), ri)
    idx, sc = rsm.route(torch.empty(0, 128, device="cuda"), 16)
    assert idx.shape == (0, 16)


# ------------------------------------------------------------------------------------ decode


@pytest.mark.parametrize("M,Dv", [(32, 64), (64, 64), (128, 128), (256, 64), (128, 96), (64, 256)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("decay", ["head", "slot"])
def test_decode_steps_match_oracle(rsm, M, Dv, dtype, decay):
    B, H, K, steps = 3, 5, min(16, M), 6
    dev = torch.device("cuda")
    st = torch.randn(B, H, M, Dv, generator=torch.Generator(device=dev).manual_seed(1), device=dev)
    ref_state = st.double().cpu().numpy()
    for s in range(steps):
        x = make_inputs(B, 1, H, M, Dv, dtype, decay, seed=1000 + s, device=dev)
        x = {n: t[:, 0].contiguous() for n, t in x.items()}
        before = st.clone()
        d = rsm.decode_step(x["q"], x["k"], x["v"], x["logits"], x["f"], K, st, routing=True)
        torch.cuda.synchronize()
        xc = host(x)
        r = oracle.decode_step(xc["q"], xc["k"], xc["v"], xc["logits"], xc["f"], K, ref_state)
        ref_state = r["state"]
        idx = d["idx"].cpu().numpy()
        assert np.array_equal(idx, r["idx"])
        assert rel(d["o"].cpu().numpy(), r["o"]) <= TOL_FP32
        assert rel(st.cpu().numpy(), ref_state) <= TOL_FP32
        # rows not selected at this step keep their bits
        sel = np.zeros((B, H, M), bool)
        np.put_along_axis(sel, idx.astype(np.int64), True, axis=2)
        nb = before.cpu().numpy().view(np.uint32)
        na = st.cpu().numpy().view(np.uint32)
        assert np.array_equal(na[~sel], nb[~sel])


# ------------------------------------------------------------------------------------ prefill


PATHS = ["simt", "auto", "tensor"]


def tensor_ok(path, M, Dv, dtype, K=16):
    """The tensor-core path covers bf16 q/k/v with M = Dv = 128 and K <= 32."""
    return path != "tensor" or (M == 128 and Dv == 128 and dtype == torch.bfloat16 and K <= 32)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("M,K,Dv,T", [(32, 4, 32, 70), (64, 16, 64, 129), (128, 16, 128, 200),
                                      (256, 32, 64, 77), (128, 1, 96, 64), (64, 64, 64, 90)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("decay", ["head", "slot"])
def test_forward_matches_oracle(rsm, path, M, K, Dv, T, dtype, decay):
    if not tensor_ok(path, M, Dv, dtype, K):
        pytest.skip("shape not on the tensor-core path")
    B, H = 2, 3
    x = make_inputs(B, T, H, M, Dv, dtype, decay, seed=M + K + T, device="cuda", h0=True)
    out = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, x["H0"], routing=True, path=path)
    torch.cuda.synchronize()
    c = host(x)
    r = oracle.forward(c["q"], c["k"], c["v"], c["logits"], c["f"], K, c["H0"])
    assert np.array_equal(out["idx"].cpu().numpy(), r["idx"])
    assert float(np.max(np.abs(out["score"].cpu().numpy() - r["score"]))) <= 1e-6
    tol = tol_for(path, dtype)
    assert rel(out["o"].cpu().numpy(), r["o"]) <= tol
    assert rel(out["HT"].cpu().numpy(), r["HT"]) <= tol


@pytest.mark.parametrize("path", PATHS)
def test_forward_zero_tokens_and_one_token(rsm, path):
    B, H, M, K, Dv = 2, 2, 128, 16, 128
    x = make_inputs(B, 1, H, M, Dv, torch.bfloat16, "head", seed=3, device="cuda", h0=True)
    e = rsm.forward(x["q"][:, :0], x["k"][:, :0], x["v"][:, :0], x["logits"][:, :0], x["f"][:, :0],
                    K, x["H0"], path=path)
    torch.cuda.synchronize()
    assert torch.equal(e["HT"], x["H0"])
    out = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, x["H0"], path=path)
    torch.cuda.synchronize()
    c = host(x)
    r = oracle.forward(c["q"], c["k"], c["v"], c["logits"], c["f"], K, c["H0"])
    tol = tol_for(path, torch.bfloat16)
    assert rel(out["o"].cpu().numpy(), r["o"]) <= tol
    assert rel(out["HT"].cpu().numpy(), r["HT"]) <= tol


@pytest.mark.parametrize("path", PATHS)
def test_forward_state_aliasing_and_resume(rsm, path):
    B, T, H, M, K, Dv = 2, 300, 2, 128, 16, 128
    x = make_inputs(B, T, H, M, Dv, torch.bfloat16, "slot", seed=8, device="cuda", h0=True)
    full = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, x["H0"], path=path)
    st = x["H0"].clone()
    cut = 137
    parts = []
    for a, b in ((0, cut), (cut, T)):
        sl = {n: x[n][:, a:b].contiguous() for n in ("q", "k", "v", "logits", "f")}
        p = rsm.forward(sl["q"], sl["k"], sl["v"], sl["logits"], sl["f"], K, st, path=path,
                        out={"HT": st})   # H0 aliases HT: the state is carried in place
        parts.append(p["o"])
    torch.cuda.synchronize()
    o2 = torch.cat(parts, dim=1)
    tol = tol_for(path, torch.bfloat16)
    assert rel(o2.cpu().numpy(), full["o"].cpu().numpy()) <= tol
    assert rel(st.cpu().numpy(), full["HT"].cpu().numpy()) <= tol


@pytest.mark.parametrize("path", PATHS)
def test_forward_unselected_slots_keep_bits(rsm, path):
    B, T, H, M, K, Dv = 1, 256, 2, 128, 16, 128
    x = make_inputs(B, T, H, M, Dv, torch.bfloat16, "head", seed=9, device="cuda", h0=True)
    x["logits"][..., M // 2:] = -100.0
    out = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, x["H0"], path=path)
    torch.cuda.synchronize()
    a = out["HT"][:, :, M // 2:].cpu().numpy().view(np.uint32)
    b = x["H0"][:, :, M // 2:].cpu().numpy().view(np.uint32)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("M,Dv", [(64, 64), (128, 128)])
def test_forward_window_limit(rsm, path, M, Dv):
    """K=1, a one-hot cyclic router and f = -1e4: the slot store becomes a window of the last M
    tokens, o_t = sum_{s=t-M+1..t} q_{t, s mod M} v_s (exercises extreme decays)."""
    if not tensor_ok(path, M, Dv, torch.bfloat16, 1):
        pytest.skip("shape not on the tensor-core path")
    B, T, H = 1, 300, 2
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(4)
    q = torch.randn(B, T, H, M, generator=g, device=dev).bfloat16()
    v = torch.randn(B, T, H, Dv, generator=g, device=dev).bfloat16()
    k = torch.ones(B, T, H, M, device=dev).bfloat16()
    logits = torch.zeros(B, T, H, M, device=dev)
    t = torch.arange(T, device=dev)
    logits[:, t, :, t % M] = 10.0
    f = torch.full((B, T, H), -1e4, device=dev)
    out = rsm.forward(q, k, v, logits, f, 1, path=path)
    torch.cuda.synchronize()
    from oracle import brute
    qc, vc = q.float().cpu().numpy(), v.float().cpu().numpy()
    for h in range(H):
        ow, HTw = brute.window_form(qc[0, :, h], vc[0, :, h], M)
        assert rel(out["o"][0, :, h].cpu().numpy(), ow) <= TOL_FP32
        assert rel(out["HT"][0, h].cpu().numpy(), HTw) <= TOL_FP32


# ------------------------------------------------------------------------------------ workloads


@pytest.mark.parametrize("name", ["tiny_fp32", "small_bf16", "mid_gla_bf16", "long_ctx_bf16"])
def test_workload_parity(rsm, name):
    """The four prefill workloads at full size, in the configuration the benchmark times."""
    w = WORKLOADS[name]
    x = make_workload_inputs(w, device="cuda")
    out = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], w.K, routing=True)
    torch.cuda.synchronize()
    c = host(x)
    r = oracle.forward(c["q"], c["k"], c["v"], c["logits"], c["f"], w.K)
    assert np.array_equal(out["idx"].cpu().numpy(), r["idx"])
    tol = TOL_FP32 if w.dtype == "f32" else TOL_BF16
    eo, eh = rel(out["o"].cpu().numpy(), r["o"]), rel(out["HT"].cpu().numpy(), r["HT"])
    print(f"{name}: o {eo:.3e} H_T {eh:.3e}")
    assert eo <= tol and eh <= tol
    # the benchmark's call: no routing outputs (the routing records then hold the selected set
    # without ranking it)
    out2 = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], w.K)
    torch.cuda.synchronize()
    assert rel(out2["o"].cpu().numpy(), r["o"]) <= tol and rel(out2["HT"].cpu().numpy(), r["HT"]) <= tol


# ------------------------------------------------------------------------------------ tensor path


@pytest.mark.parametrize("T", [1000, 4096 + 77])
@pytest.mark.parametrize("decay", ["head", "slot"])
def test_tensor_segments_match_oracle(rsm, T, decay):
    """Few (b,h) streams and a long sequence: the sequence is split into segments (segment
    summaries, scan of segment states, chunk scan). Random initial state."""
    B, H, M, K, Dv = 1, 2, 128, 16, 128
    x = make_inputs(B, T, H, M, Dv, torch.bfloat16, decay, seed=T, device="cuda", h0=True)
    out = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, x["H0"], routing=True, path="tensor")
    torch.cuda.synchronize()
    c = host(x)
    r = oracle.forward(c["q"], c["k"], c["v"], c["logits"], c["f"], K, c["H0"])
    assert np.array_equal(out["idx"].cpu().numpy(), r["idx"])
    eo, eh = rel(out["o"].cpu().numpy(), r["o"]), rel(out["HT"].cpu().numpy(), r["HT"])
    print(f"T={T} {decay}: o {eo:.3e} H_T {eh:.3e}")
    assert eo <= TOL_BF16 and eh <= TOL_BF16


def test_tensor_segments_with_aliased_state(rsm):
    """H0 and HT are the same buffer while several segments run in parallel."""
    B, T, H, M, K, Dv = 1, 1500, 2, 128, 16, 128
    x = make_inputs(B, T, H, M, Dv, torch.bfloat16, "head", seed=77, device="cuda", h0=True)
    c = host(x)
    st = x["H0"].clone()
    out = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, st, path="tensor", out={"HT": st})
    torch.cuda.synchronize()
    r = oracle.forward(c["q"], c["k"], c["v"], c["logits"], c["f"], K, c["H0"])
    assert rel(out["o"].cpu().numpy(), r["o"]) <= TOL_BF16
    assert rel(st.cpu().numpy(), r["HT"]) <= TOL_BF16


def test_tensor_segments_unselected_slots_keep_bits(rsm):
    """A long sequence split into segments: slots that no token selects pass the initial state
    through every segment summary (D = 1, U = 0) and the scan bit for bit."""
    B, T, H, M, K, Dv = 1, 4096 + 77, 2, 128, 16, 128
    x = make_inputs(B, T, H, M, Dv, torch.bfloat16, "head", seed=19, device="cuda", h0=True)
    x["logits"][..., M // 2:] = -100.0
    out = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, x["H0"], path="tensor")
    torch.cuda.synchronize()
    a = out["HT"][:, :, M // 2:].cpu().numpy().view(np.uint32)
    b = x["H0"][:, :, M // 2:].cpu().numpy().view(np.uint32)
    assert np.array_equal(a, b)


def test_tensor_segments_window_limit(rsm):
    """The window-limit case (K=1, one-hot cyclic router, f = -1e4) over a sequence long enough to
    be split into segments: the segment summaries see decays of e^-10000 and still give the window
    form o_t = sum_{s=t-M+1..t} q_{t, s mod M} v_s."""
    B, T, H, M, Dv = 1, 2000, 2, 128, 128
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(6)
    q = torch.randn(B, T, H, M, generator=g, device=dev).bfloat16()
    v = torch.randn(B, T, H, Dv, generator=g, device=dev).bfloat16()
    k = torch.ones(B, T, H, M, device=dev).bfloat16()
    logits = torch.zeros(B, T, H, M, device=dev)
    t = torch.arange(T, device=dev)
    logits[:, t, :, t % M] = 10.0
    f = torch.full((B, T, H), -1e4, device=dev)
    out = rsm.forward(q, k, v, logits, f, 1, path="tensor")
    torch.cuda.synchronize()
    from oracle import brute
    qc, vc = q.float().cpu().numpy(), v.float().cpu().numpy()
    for h in range(H):
        ow, HTw = brute.window_form(qc[0, :, h], vc[0, :, h], M)
        assert rel(out["o"][0, :, h].cpu().numpy(), ow) <= TOL_FP32
        assert rel(out["HT"][0, h].cpu().numpy(), HTw) <= TOL_FP32


def test_tensor_mixed_fast_and_exact_chunks(rsm):
    """Some tokens forget almost everything (f = -1e4): their chunks take the exact path while
    the others take the tensor-core path; results still match the oracle."""
    B, T, H, M, K, Dv = 2, 700, 2, 128, 16, 128
    x = make_inputs(B, T, H, M, Dv, torch.bfloat16, "head", seed=5, device="cuda", h0=True)
    x["f"][:, 100:110] = -1e4
    x["f"][:, 333] = -200.0
    out = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, x["H0"], path="tensor")
    torch.cuda.synchronize()
    c = host(x)
    r = oracle.forward(c["q"], c["k"], c["v"], c["logits"], c["f"], K, c["H0"])
    eo, eh = rel(out["o"].cpu().numpy(), r["o"]), rel(out["HT"].cpu().numpy(), r["HT"])
    print(f"mixed: o {eo:.3e} H_T {eh:.3e}")
    assert eo <= TOL_BF16 and eh <= TOL_BF16


def test_tensor_path_is_selected_for_supported_shapes(rsm):
    from sparse_routed_slot_b200 import api
    x = make_inputs(1, 64, 1, 128, 128, torch.bfloat16, "head", seed=1, device="cuda")
    o = torch.empty(1, 64, 1, 128, device="cuda")
    a = api._forward_args(x["q"], x["k"], x["v"], x["logits"], x["f"], 16, None, o, None, None, None,
                          "auto", False)
    assert api.selected_path(a) == "tensor"
    y = make_inputs(1, 64, 1, 128, 128, torch.float32, "head", seed=1, device="cuda")
    a = api._forward_args(y["q"], y["k"], y["v"], y["logits"], y["f"], 16, None, o, None, None, None,
                          "auto", False)
    assert api.selected_path(a) == "simt"


def test_forward_profile_events_split_the_call(rsm):
    """rsm_forward_set_profile_events: one event before the first kernel and one after each; the
    per-kernel times add up to the whole call, and results are unchanged."""
    import ctypes
    from sparse_routed_slot_b200 import _lib, api
    B, T, H, M, K, Dv = 1, 3000, 2, 128, 16, 128
    x = make_inputs(B, T, H, M, Dv, torch.bfloat16, "head", seed=31, device="cuda")
    ref = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], K)
    o = torch.empty_like(ref["o"])
    HT = torch.empty_like(ref["HT"])
    a = api._forward_args(x["q"], x["k"], x["v"], x["logits"], x["f"], K, None, o, HT, None, None, "auto", False)
    n = api.kernel_launches(a)
    assert n >= 2
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
    for e in ev:
        e.record(stream)  # creates the CUDA events
    torch.cuda.synchronize()
    L = _lib.load()
    ptrs = (ctypes.c_void_p * (n + 1))(*[e.cuda_event for e in ev])
    _lib.check(L.rsm_forward_set_profile_events(ptrs, n + 1))
    try:
        rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, out={"o": o, "HT": HT})
    finally:
        _lib.check(L.rsm_forward_set_profile_events(None, 0))
    torch.cuda.synchronize()
    parts = [ev[i].elapsed_time(ev[i + 1]) for i in range(n)]
    assert all(p > 0 for p in parts)
    assert abs(sum(parts) - ev[0].elapsed_time(ev[n])) < 1e-3
    assert torch.equal(o, ref["o"]) and torch.equal(HT, ref["HT"])


@pytest.mark.parametrize("M,Dv", [(32, 4), (64, 12), (128, 20), (256, 36)])
def test_simt_narrow_and_ragged_value_tiles(rsm, M, Dv):
    """The CUDA-core path works in value-column tiles of 64 (32 at M = 256); narrower value
    widths and ragged last tiles are masked."""
    B, T, H, K = 2, 75, 2, min(16, M)
    x = make_inputs(B, T, H, M, Dv, torch.float32, "slot", seed=M + Dv, device="cuda", h0=True)
    out = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, x["H0"], path="simt")
    torch.cuda.synchronize()
    c = host(x)
    r = oracle.forward(c["q"], c["k"], c["v"], c["logits"], c["f"], K, c["H0"])
    assert rel(out["o"].cpu().numpy(), r["o"]) <= TOL_FP32
    assert rel(out["HT"].cpu().numpy(), r["HT"]) <= TOL_FP32


@pytest.mark.parametrize("M", [32, 64, 128])
@pytest.mark.parametrize("K", [2, 8, 16, 31])
def test_simt_set_selection_with_ties(rsm, M, K):
    """Without ranked outputs the CUDA-core path takes each row's TopK set from a threshold search
    seeded with the previous row, and the ranking tournament where the search meets a tie at the
    cut. Logit rows with many exact ties, one-ulp near ties and plain Gaussian rows (so both ways
    run, and the seed jumps between distributions): the per-slot selection counts, which fix every
    row's set, are bit-exact, and o and the state match at the fp32 bar."""
    B, T, H, Dv = 1, 96, 2, 64
    x = make_inputs(B, T, H, M, Dv, torch.float32, "slot", seed=M * 7 + K, device="cuda", h0=True)
    g = torch.Generator().manual_seed(M + K)
    lg = torch.randn(B, T, H, M, generator=g)
    lg[:, 16:48] = torch.round(3 * torch.randn(B, 32, H, M, generator=g)) / 3        # exact ties
    near = torch.full((B, 16, H, M), 0.75)
    bump = torch.rand(B, 16, H, M, generator=g) < 0.5
    near[bump] = torch.nextafter(torch.tensor(0.75), torch.tensor(1.0))
    lg[:, 48:64] = near                                                                # near ties
    x["logits"] = lg.float().contiguous().cuda()
    counts = torch.zeros((B, H, M), dtype=torch.int32, device="cuda")
    out = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, x["H0"], path="simt", slot_counts=counts)
    torch.cuda.synchronize()
    c = host(x)
    r = oracle.forward(c["q"], c["k"], c["v"], c["logits"], c["f"], K, c["H0"], want_counts=True)
    assert np.array_equal(counts.cpu().numpy(), r["counts"])
    assert rel(out["o"].cpu().numpy(), r["o"]) <= TOL_FP32
    assert rel(out["HT"].cpu().numpy(), r["HT"]) <= TOL_FP32
