"""GPU parity of the persistent kernels at shapes where every CTA walks several (b,h) items.

The chunk scan and the decode kernel run one persistent CTA per SM; with more (b,h) streams than
SMs a CTA finishes one stream's state and starts the next one's inside the same launch (the
decode kernel's state ring and routing-slot ring wrap across items). These tests compare those
paths with the fp64 oracle:

* the tensor-core prefill that builds the generation workload's state (32 sequences x 16 heads x
  2048 tokens per call: 512 streams over the SMs, about 3.5 per CTA);
* the generation workload itself: 256 sequences x 16 heads (4096 streams, about 28 per CTA),
  M = 128, K = 16, Dv = 128, bf16 q/k/v, state from that prefill, all 1024 steps, on sequences
  {0, 127, 255} x all heads: indices bit-exact, o and the state at the fp32 bar every step, and
  the rows not selected at a step keep their bits;
* a few decode steps with 1024 streams at M = Dv = 128 and M = Dv = 256 (six routing slots) on
  every stream.
"""
import numpy as np
import pytest
import torch

from oracle import oracle
from sparse_routed_slot_b200.workloads import (DECODE_PREFILL_GROUP, WORKLOADS, decode_prefill_group,
                                               decode_step_inputs, make_inputs)

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


def sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def test_chunk_scan_several_streams_per_cta(rsm):
    """One prefill call of the decode workload's set-up (the benchmark's call): 512 streams, so
    each persistent CTA of the chunk scan carries state out of one stream and into the next.
    Sequences 0, 9, 15, 18 and 31 cover the first stream of CTAs and streams 147/148 and 295/296,
    where the walk crosses the grid."""
    w = WORKLOADS["decode_256x16"]
    x = decode_prefill_group(w, 0, device="cuda")
    assert DECODE_PREFILL_GROUP * w.H > 3 * sms()
    out = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], w.K, routing=True, path="tensor")
    torch.cuda.synchronize()
    seqs = [0, 9, 15, 18, 31]
    c = {n: t[seqs].float().cpu().numpy() for n, t in x.items()}
    r = oracle.forward(c["q"], c["k"], c["v"], c["logits"], c["f"], w.K)
    assert np.array_equal(out["idx"][seqs].cpu().numpy(), r["idx"])
    eo = rel(out["o"][seqs].cpu().numpy(), r["o"])
    eh = rel(out["HT"][seqs].cpu().numpy(), r["HT"])
    print(f"32x16 streams x 2048 tokens: o {eo:.3e} H_T {eh:.3e}")
    assert eo <= TOL_BF16 and eh <= TOL_BF16


def _decode_state(rsm, w, seqs):
    """The generation workload's state (all sequences) built as the benchmark builds it, and the
    oracle's prefill of the checked sequences."""
    state = torch.zeros(w.B, w.H, w.M, w.Dv, dtype=torch.float32, device="cuda")
    ref = {}
    for b0 in range(0, w.B, DECODE_PREFILL_GROUP):
        x = decode_prefill_group(w, b0, device="cuda")
        out = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], w.K, state=True)
        state[b0:b0 + DECODE_PREFILL_GROUP].copy_(out["HT"])
        local = [s - b0 for s in seqs if b0 <= s < b0 + DECODE_PREFILL_GROUP]
        if local:
            c = {n: t[local].float().cpu().numpy() for n, t in x.items()}
            r = oracle.forward(c["q"], c["k"], c["v"], c["logits"], c["f"], w.K, want_idx=False)
            for j, s in enumerate(local):
                ref[b0 + s] = r["HT"][j]
        del x, out
    torch.cuda.synchronize()
    return state, np.stack([ref[s] for s in seqs])


def test_decode_workload_all_steps(rsm):
    """256 sequences x 16 heads, state from the 2048-token prefill, 1024 steps (the generation
    workload as the benchmark runs it), checked on sequences 0, 127 and 255 at every step."""
    w = WORKLOADS["decode_256x16"]
    seqs = [0, 127, 255]
    state, ref_prefill = _decode_state(rsm, w, seqs)
    e_pre = rel(state[seqs].cpu().numpy(), ref_prefill)
    print(f"prefill state (tensor path) vs oracle: {e_pre:.3e}")
    assert e_pre <= TOL_BF16
    d = decode_step_inputs(w, w.decode_steps, device="cuda")
    dc = {n: t[:, seqs].float().cpu().numpy() for n, t in d.items()}
    # the oracle continues from the device's post-prefill state, so the decode is checked alone
    ref_state = state[seqs].double().cpu().numpy()
    o = torch.empty(w.B, w.H, w.Dv, device="cuda")
    worst_o = worst_s = 0.0
    for i in range(w.decode_steps):
        before = state[seqs].cpu().numpy()
        res = rsm.decode_step(d["q"][i], d["k"][i], d["v"][i], d["logits"][i], d["f"][i], w.K, state,
                              routing=True, o=o)
        r = oracle.decode_step(dc["q"][i], dc["k"][i], dc["v"][i], dc["logits"][i], dc["f"][i], w.K,
                               ref_state)
        ref_state = r["state"]
        idx = res["idx"][seqs].cpu().numpy()
        assert np.array_equal(idx, r["idx"]), f"step {i}: indices"
        after = state[seqs].cpu().numpy()
        eo, es = rel(o[seqs].cpu().numpy(), r["o"]), rel(after, ref_state)
        worst_o, worst_s = max(worst_o, eo), max(worst_s, es)
        assert eo <= TOL_FP32 and es <= TOL_FP32, f"step {i}: o {eo:.2e} state {es:.2e}"
        sel = np.zeros((len(seqs), w.H, w.M), bool)
        np.put_along_axis(sel, idx.astype(np.int64), True, axis=2)
        assert np.array_equal(after.view(np.uint32)[~sel], before.view(np.uint32)[~sel]), f"step {i}"
    print(f"1024 decode steps: worst o {worst_o:.3e} state {worst_s:.3e}")


@pytest.mark.parametrize("M,Dv", [(128, 128), (256, 256)])
def test_decode_several_streams_per_cta(rsm, M, Dv):
    """1024 streams (about 7 per CTA): every stream checked for a few steps."""
    B, H, K, steps = 64, 16, 16, 3
    assert B * H > 3 * sms()
    dev = torch.device("cuda")
    st = torch.randn(B, H, M, Dv, generator=torch.Generator(device=dev).manual_seed(5), device=dev)
    ref_state = st.double().cpu().numpy()
    for s in range(steps):
        x = make_inputs(B, 1, H, M, Dv, torch.bfloat16, "head", seed=500 + s, device=dev)
        x = {n: t[:, 0].contiguous() for n, t in x.items()}
        before = st.cpu().numpy()
        res = rsm.decode_step(x["q"], x["k"], x["v"], x["logits"], x["f"], K, st, routing=True)
        torch.cuda.synchronize()
        xc = {n: t.float().cpu().numpy() for n, t in x.items()}
        r = oracle.decode_step(xc["q"], xc["k"], xc["v"], xc["logits"], xc["f"], K, ref_state)
        ref_state = r["state"]
        idx = res["idx"].cpu().numpy()
        assert np.array_equal(idx, r["idx"])
        after = st.cpu().numpy()
        assert rel(res["o"].cpu().numpy(), r["o"]) <= TOL_FP32
        assert rel(after, ref_state) <= TOL_FP32
        sel = np.zeros((B, H, M), bool)
        np.put_along_axis(sel, idx.astype(np.int64), True, axis=2)
        assert np.array_equal(after.view(np.uint32)[~sel], before.view(np.uint32)[~sel])
