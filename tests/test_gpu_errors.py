"""Error paths on the GPU, made on the host (nothing here faults, traps or hangs a device).

* RSM_FLAG_VALIDATE: a non-finite logit, or a positive or non-finite log-decay f, is reported by
  rsm_get_device_status as RSM_ERR_NONFINITE after rsm_forward (both paths) and rsm_decode_step;
  valid inputs report RSM_OK, and the status word is cleared by the read.
* Bounded waits: RSM_FLAG_TEST_STALL_ROUTING makes the decode kernel's routing warps hand over
  nothing, so the consumer warps' wait for a routing slot expires after a short bound; the call
  reports RSM_ERR_TIMEOUT, leaves o and the state unwritten, and the context stays usable (a
  normal step afterwards matches the oracle). With the same flag rsm_backward withholds its first
  token's copy and bounds its waits to one poll: the first wait expires with the next tokens' copies
  in flight, the kernel drains them and reports RSM_ERR_TIMEOUT, and a normal call afterwards
  matches the oracle.
"""
import numpy as np
import pytest
import torch

from oracle import oracle
from sparse_routed_slot_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rsm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    import sparse_routed_slot_b200 as m
    from sparse_routed_slot_b200 import _lib
    m.device_status()  # start from a clear status word
    return m, _lib


def rel(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(x - ref)) / max(np.sqrt(np.mean(ref ** 2)), 1e-300))


def _spoil(x, what, decay):
    x = {n: t.clone() for n, t in x.items()}
    if what == "nan_logit":
        x["logits"].view(-1)[37] = float("nan")
    elif what == "inf_logit":
        x["logits"].view(-1)[-5] = float("inf")
    elif what == "positive_f":
        x["f"].view(-1)[3] = 0.25
    elif what == "nan_f":
        x["f"].view(-1)[-1] = float("nan")
    return x


BAD = ["nan_logit", "inf_logit", "positive_f", "nan_f"]


@pytest.mark.parametrize("path", ["simt", "tensor"])
@pytest.mark.parametrize("decay", ["head", "slot"])
@pytest.mark.parametrize("what", ["ok"] + BAD)
def test_forward_validate(rsm, path, decay, what):
    m, lib = rsm
    x = make_inputs(1, 150, 2, 128, 128, torch.bfloat16, decay, seed=3, device="cuda")
    x = _spoil(x, what, decay)
    m.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], 16, path=path, validate=True)
    status = m.device_status()
    assert status == (lib.RSM_OK if what == "ok" else lib.RSM_ERR_NONFINITE)
    assert m.device_status() == lib.RSM_OK  # reading clears it


@pytest.mark.parametrize("decay", ["head", "slot"])
@pytest.mark.parametrize("what", ["ok"] + BAD)
def test_decode_validate(rsm, decay, what):
    m, lib = rsm
    x = make_inputs(3, 1, 4, 128, 64, torch.bfloat16, decay, seed=4, device="cuda")
    x = {n: t[:, 0].contiguous() for n, t in x.items()}
    x = _spoil(x, what, decay)
    st = torch.zeros(3, 4, 128, 64, device="cuda")
    m.decode_step(x["q"], x["k"], x["v"], x["logits"], x["f"], 16, st, validate=True)
    assert m.device_status() == (lib.RSM_OK if what == "ok" else lib.RSM_ERR_NONFINITE)


def test_forward_without_validate_reports_nothing(rsm):
    m, lib = rsm
    x = _spoil(make_inputs(1, 64, 1, 128, 128, torch.bfloat16, "head", seed=5, device="cuda"), "positive_f", "head")
    m.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], 16)
    assert m.device_status() == lib.RSM_OK


def test_decode_routing_stall_times_out_and_context_survives(rsm):
    m, lib = rsm
    B, H, M, K, Dv = 40, 16, 128, 16, 128  # 640 streams: several per CTA
    x = make_inputs(B, 1, H, M, Dv, torch.bfloat16, "head", seed=6, device="cuda")
    x = {n: t[:, 0].contiguous() for n, t in x.items()}
    st = torch.randn(B, H, M, Dv, generator=torch.Generator(device="cuda").manual_seed(2), device="cuda")
    st0 = st.clone()
    o = torch.full((B, H, Dv), float("nan"), device="cuda")
    m.decode_step(x["q"], x["k"], x["v"], x["logits"], x["f"], K, st, o=o, flags=lib.RSM_FLAG_TEST_STALL_ROUTING)
    assert m.device_status() == lib.RSM_ERR_TIMEOUT
    assert torch.equal(st, st0)          # no row was written
    assert torch.isnan(o).all()          # no output was written
    assert m.device_status() == lib.RSM_OK
    # the context is still usable: the same step without the flag matches the oracle
    res = m.decode_step(x["q"], x["k"], x["v"], x["logits"], x["f"], K, st, routing=True)
    assert m.device_status() == lib.RSM_OK
    xc = {n: t.float().cpu().numpy() for n, t in x.items()}
    r = oracle.decode_step(xc["q"], xc["k"], xc["v"], xc["logits"], xc["f"], K, st0.double().cpu().numpy())
    assert np.array_equal(res["idx"].cpu().numpy(), r["idx"])
    assert rel(res["o"].cpu().numpy(), r["o"]) <= 1e-4
    assert rel(st.cpu().numpy(), r["state"]) <= 1e-4


def test_backward_wait_expiry_reports_timeout_and_drains(rsm):
    m, lib = rsm
    B, T, H, M, K, Dv = 1, 40, 2, 64, 8, 64
    x = make_inputs(B, T, H, M, Dv, torch.float32, "head", seed=5, device="cuda")
    dO = torch.randn(B, T, H, Dv, generator=torch.Generator(device="cuda").manual_seed(4), device="cuda")
    m.backward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, dO, None, flags=lib.RSM_FLAG_TEST_STALL_ROUTING)
    torch.cuda.synchronize()
    assert m.device_status() == lib.RSM_ERR_TIMEOUT
    assert m.device_status() == lib.RSM_OK
    # the context is still usable: the same call without the flag matches the oracle
    out = m.backward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, dO, None)
    torch.cuda.synchronize()
    assert m.device_status() == lib.RSM_OK
    c = {n: t.float().cpu().numpy() for n, t in x.items()}
    r = oracle.backward(c["q"], c["k"], c["v"], c["logits"], c["f"], K, dO=dO.cpu().numpy())
    for n in ("dq", "dk", "dv", "dlogits", "df", "dH0"):
        assert rel(out[n].cpu().numpy(), r[n]) <= 1e-4, n
