"""Host logic of the profiling case: reading ncu's CSV and summarising DRAM bytes per call."""

import json

import pytest

from sparse_routed_slot_b200 import profile_case as pc

HEADER = ['"ID"', '"Process ID"', '"Process Name"', '"Host Name"', '"Kernel Name"', '"Context"', '"Stream"',
          '"Block Size"', '"Grid Size"', '"Device"', '"CC"', '"Section Name"', '"Metric Name"', '"Metric Unit"',
          '"Metric Value"']


def _csv(tmp_path, launches):
    """launches: [(kernel name, {metric: value})] -> an ncu --csv log with a preamble line."""
    lines = ["==PROF== Connected to process 1", ",".join(HEADER)]
    for i, (name, metrics) in enumerate(launches):
        for m, v in metrics.items():
            row = [str(i), "1", "python", "h", f"{name}(Params)", "1", "7", "(128, 1, 1)", "(148, 1, 1)", "0", "10.0",
                   "Command line profiler metrics", m, "byte", f"{v:,}"]
            lines.append(",".join(f'"{c}"' for c in row))
    p = tmp_path / "t.csv"
    p.write_text("\n".join(lines) + "\n")
    return str(p)


def _m(r, w, ns=1000):
    return {"dram__bytes_read.sum": r, "dram__bytes_write.sum": w, "gpu__time_duration.sum": ns}


def test_summary_takes_the_last_forward_and_decode_step(tmp_path):
    fwd = ["void rsm::route_rec_kernel<16, 0>", "void rsm::segment_summary_kernel<16>",
           "rsm::segment_scan_kernel", "void rsm::prefill_tc_kernel<16>"]
    launches = [("at::normal_kernel", _m(5, 5))]
    launches += [(n, _m(100 + i, 10)) for i, n in enumerate(fwd)]       # first forward
    launches += [(n, _m(1000 + i, 20)) for i, n in enumerate(fwd)]      # second forward
    launches += [("void rsm::decode_kernel<128, bf16>", _m(7, 1)), ("void rsm::decode_kernel<128, bf16>", _m(9, 3))]
    out = tmp_path / "traffic.json"
    d = pc.summarize_traffic(_csv(tmp_path, launches), "wl", str(out))
    assert d["bytes"]["wl/forward"] == sum(1000 + i + 20 for i in range(4))
    assert d["bytes"]["decode_256x16/step"] == 12
    assert json.loads(out.read_text())["sources_sha256"] == pc.sources_digest()
    assert set(d["per_kernel"]) == set(fwd) | {"void rsm::decode_kernel<128, bf16>"}


def test_summary_of_a_two_launch_forward(tmp_path):
    # an unsegmented forward is routing records + chunk scan; two forwards back to back
    fwd = ["void rsm::route_rec_kernel<16, 0>", "void rsm::prefill_tc_kernel<16>"]
    launches = [(n, _m(10 * (i + 1), 1)) for i, n in enumerate(fwd)] + [(n, _m(300 + i, 2)) for i, n in enumerate(fwd)]
    d = pc.summarize_traffic(_csv(tmp_path, launches), "wl", str(tmp_path / "o.json"))
    assert d["bytes"]["wl/forward"] == 300 + 301 + 4
    assert d["bytes"]["decode_256x16/step"] == 0


def test_reader_rejects_a_log_without_metrics(tmp_path):
    p = tmp_path / "empty.csv"
    p.write_text("==PROF== nothing here\n")
    with pytest.raises(StopIteration):
        pc.read_ncu_csv(str(p))
