"""Profiling case for ncu, and the summary of its DRAM counters.

Run a fixed case through the public API (on cuda:0, synthetic inputs):

    python -m sparse_routed_slot_b200.profile_case run [--workload long_ctx_bf16] [--forwards 2]
                                                      [--decode-steps 2] [--tokens T]

--tokens replaces the workload's sequence length (a smaller case of the same kernels, for captures
that replay each launch many times).

Each forward makes rsm_forward_kernel_launches() launches (routing records, segment summary,
segment scan, chunk scan on the tensor path); the decode steps use decode_256x16. These three
metrics take one pass (check on one launch of a --tokens case first: ncu prints "- 1 pass"), so
the full-size case can be captured, limited to the launches that are read (the second forward and
the two decode steps):

    ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum \\
        --clock-control none -k regex:"route_rec|segment_summary|segment_scan|prefill_tc|decode_kernel" \\
        -s 4 -c 6 --csv --log-file traffic.csv python -m sparse_routed_slot_b200.profile_case run

then write the per-call DRAM bytes of the LAST forward and the LAST decode step, keyed to the
current CUDA sources, to profiles/traffic.json:

    python -m sparse_routed_slot_b200.profile_case traffic traffic.csv

Section captures of one kernel each on a smaller case (--tokens) add the tensor-pipe activity:

    ncu --section SpeedOfLight ... --clock-control none -k regex:prefill_tc_kernel -s 1 -c 1 \
        -o prof_tc python -m sparse_routed_slot_b200.profile_case run --tokens 8192 --decode-steps 0
    ncu -i prof_tc.ncu-rep --page raw --csv > prof_tc.csv
    python -m sparse_routed_slot_b200.profile_case pipes prof_tc.csv [more.csv ...]

bench.py reads that file and reports its figures only while the sources still hash the same.
"""

from __future__ import annotations

import argparse
import collections
import csv
import glob
import hashlib
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FORWARD_KERNELS = ("route_rec_kernel", "segment_summary_kernel", "segment_scan_kernel", "prefill_tc_kernel",
                   "prefill_simt_kernel")
DECODE_KERNELS = ("decode_kernel",)


def sources_digest() -> str:
    """sha256 of the CUDA sources (the key under which measured counters stay valid)."""
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "sparse_routed_slot_b200", "csrc", "*"))):
        h.update(open(f, "rb").read())
    return h.hexdigest()


def run_case(workload: str, forwards: int, decode_steps: int, tokens: int = 0) -> None:
    import torch

    import sparse_routed_slot_b200 as rsm
    from sparse_routed_slot_b200.workloads import WORKLOADS, make_inputs

    dev = torch.device("cuda", 0)
    w = WORKLOADS[workload]
    T = tokens if tokens > 0 else w.T
    x = make_inputs(w.B, T, w.H, w.M, w.Dv, w.torch_dtype, w.decay, seed=w.seed, device=dev)
    for _ in range(forwards):
        out = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], w.K)
    torch.cuda.synchronize()
    del x, out
    if decode_steps > 0:
        d = WORKLOADS["decode_256x16"]
        state = torch.randn(d.B, d.H, d.M, d.Dv, device=dev)
        y = make_inputs(decode_steps, d.B, d.H, d.M, d.Dv, d.torch_dtype, d.decay, seed=9, device=dev)
        for i in range(decode_steps):
            rsm.decode_step(y["q"][i], y["k"][i], y["v"][i], y["logits"][i], y["f"][i], d.K, state)
        torch.cuda.synchronize()


def read_ncu_csv(path: str):
    """[(kernel name, {metric: value})] in launch order from an ncu --csv log."""
    rows = list(csv.reader(open(path)))
    hi = next(i for i, r in enumerate(rows) if "Kernel Name" in r and "Metric Name" in r)
    h = rows[hi]
    ki, ii, mi, vi = h.index("Kernel Name"), h.index("ID"), h.index("Metric Name"), h.index("Metric Value")
    launches: "collections.OrderedDict[str, tuple]" = collections.OrderedDict()
    for r in rows[hi + 1:]:
        if len(r) <= vi:
            continue
        name, metrics = launches.setdefault(r[ii], (r[ki].split("(")[0], {}))
        metrics[r[mi]] = float(r[vi].replace(",", ""))
    return list(launches.values())


def summarize_traffic(csv_path: str, workload: str, out_path: str) -> dict:
    launches = read_ncu_csv(csv_path)

    def last_group(kinds):
        """The last maximal run of consecutive launches whose names match `kinds` (one call)."""
        idx = [i for i, (n, _) in enumerate(launches) if any(k in n for k in kinds)]
        if not idx:
            return []
        group = [idx[-1]]
        for i in reversed(idx[:-1]):
            if i != group[-1] - 1:
                break
            # a forward starts with the routing kernel: stop after including it
            if "route_rec_kernel" in launches[group[-1]][0]:
                break
            group.append(i)
        return [launches[i] for i in reversed(group)]

    fwd = last_group(FORWARD_KERNELS)
    dec = last_group(DECODE_KERNELS)[-1:]

    def total(group):
        return int(sum(m.get("dram__bytes_read.sum", 0) + m.get("dram__bytes_write.sum", 0) for _, m in group))

    per_kernel = {}
    for name, m in fwd + dec:
        per_kernel[name] = {"read": int(m.get("dram__bytes_read.sum", 0)), "write": int(m.get("dram__bytes_write.sum", 0)),
                            "ns": int(m.get("gpu__time_duration.sum", 0))}
    d = {
        "sources_sha256": sources_digest(),
        "how": ("ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum --clock-control none "
                f"python -m sparse_routed_slot_b200.profile_case run --workload {workload}; the last forward "
                f"({len(fwd)} launches, summed) and the last decode step"),
        "bytes": {f"{workload}/forward": total(fwd), "decode_256x16/step": total(dec)},
        "per_kernel": per_kernel,
    }
    with open(out_path, "w") as fh:
        json.dump(d, fh, indent=1)
        fh.write("\n")
    return d


PIPE_METRIC = "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_elapsed"


def read_ncu_raw_csv(path: str):
    """[(kernel name, {metric: value})] from `ncu -i report --page raw --csv` (one row per launch,
    one column per metric, a units row under the header)."""
    rows = list(csv.reader(open(path)))
    hi = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    h = rows[hi]
    ki = h.index("Kernel Name")
    out = []
    for r in rows[hi + 2:]:
        if len(r) != len(h):
            continue
        m = {}
        for name, val in zip(h, r):
            try:
                m[name] = float(val.replace(",", ""))
            except ValueError:
                pass
        out.append((r[ki].split("(")[0].strip(), m))
    return out


def merge_pipes(csv_paths, out_path: str) -> dict:
    """Adds each captured kernel's tensor-pipe activity (percent of elapsed cycles) to the traffic
    file, under per_kernel[name]["tensor_pipe_pct"], with the case it was measured on."""
    d = json.load(open(out_path))
    if d.get("sources_sha256") != sources_digest():
        raise SystemExit("the traffic file was recorded for other kernel sources; capture it again first")
    for p in csv_paths:
        for name, m in read_ncu_raw_csv(p):
            if PIPE_METRIC not in m:
                continue
            base = name.split("::")[-1]  # e.g. prefill_tc_kernel<16>
            key = next((k for k in d["per_kernel"] if k.split("(")[0].strip().endswith(base)), name)
            d["per_kernel"].setdefault(key, {})["tensor_pipe_pct"] = m[PIPE_METRIC]
    d["tensor_pipe_how"] = ("ncu section capture of one kernel per command (-k <kernel> -s 1 -c 1) on "
                            "profile_case run --tokens 8192")
    with open(out_path, "w") as fh:
        json.dump(d, fh, indent=1)
        fh.write("\n")
    return d


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    sub = ap.add_subparsers(dest="cmd", required=True)
    r = sub.add_parser("run")
    r.add_argument("--workload", default="long_ctx_bf16")
    r.add_argument("--forwards", type=int, default=2)
    r.add_argument("--decode-steps", type=int, default=2)
    r.add_argument("--tokens", type=int, default=0)
    t = sub.add_parser("traffic")
    t.add_argument("csv")
    t.add_argument("--workload", default="long_ctx_bf16")
    t.add_argument("--out", default=os.path.join(ROOT, "profiles", "traffic.json"))
    pp = sub.add_parser("pipes")
    pp.add_argument("csv", nargs="+")
    pp.add_argument("--out", default=os.path.join(ROOT, "profiles", "traffic.json"))
    a = ap.parse_args(argv)
    if a.cmd == "run":
        run_case(a.workload, a.forwards, a.decode_steps, a.tokens)
        print("ok")
    elif a.cmd == "pipes":
        d = merge_pipes(a.csv, a.out)
        print(json.dumps({k: v.get("tensor_pipe_pct") for k, v in d["per_kernel"].items()}))
    else:
        d = summarize_traffic(a.csv, a.workload, a.out)
        print(json.dumps(d["bytes"]))


if __name__ == "__main__":
    main()
