"""Benchmark of the RSM mixer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one chunked prefill (rsm_forward) of the chosen workload, inputs resident in HBM
(default: the 32K-token long-context prefill, B=1 T=32768 H=16 M=128 K=16 Dv=128, bf16 q/k/v,
fp32 logits/state/output). The JSON line also carries
  - `configs`: the other prefill workloads (tiny fp32 check, the pages' small training shape, the
    mid-size per-slot-decay prefill), each with its time, roofline and the oracle beside it;
  - `decode`: the generation workload (rsm_decode_step on 256 sequences x 16 heads, M=128 K=16
    Dv=128, state from a 2048-token prefill), all 1024 steps timed on the device, an end-to-end
    figure with each step's inputs copied in from host memory, and the oracle on its first steps.
Roofline bytes are the path's algorithmic bytes (o counted in v's dtype); the extra bytes of the
library's fp32 o are reported beside them.

Under torchrun (N > 1) every rank runs its own replica on its own GPU with its own inputs (the
path shards by sequence with no data exchange), timing is taken on the device with CUDA events,
and the max over ranks is reported (weak scaling). `--impl reference` times the fp64 CPU oracle
on bounded samples of the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "RSM prefill tokens/s and decode state HBM GB/s on 1 B200; % roofline"


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# --------------------------------------------------------------------------- work accounting

def prefill_bytes(w) -> int:
    """Algorithmic bytes of one prefill (the per-token-head figure of the path's scope table):
    every input read once, o written once in v's dtype, H_T written once."""
    es = 2 if w.dtype == "bf16" else 4
    th = w.B * w.T * w.H
    b = th * (2 * w.M * es + w.Dv * es + w.M * 4)          # q, k, v, logits
    b += th * (w.M * 4 if w.decay == "slot" else 4)        # f
    b += th * w.Dv * es                                    # o in v's dtype
    b += w.B * w.H * w.M * w.Dv * 4                        # H_T
    return b


def o_fp32_extra_bytes(w) -> int:
    """Bytes the library writes beyond prefill_bytes(): it returns o in fp32 for every input dtype
    (a bf16 o alone would take most of the bf16 error bar on heavy-tailed outputs)."""
    es = 2 if w.dtype == "bf16" else 4
    return w.B * w.T * w.H * w.Dv * (4 - es)


def prefill_flops(w, chunk=64) -> int:
    """Dense-contraction FLOPs of the chunked form: 4*M*Dv + 2*C*(M+Dv) per token-head."""
    return w.B * w.T * w.H * (4 * w.M * w.Dv + 2 * chunk * (w.M + w.Dv))


def decode_bytes(B, H, M, K, Dv, es=2, per_slot=False) -> tuple[int, int]:
    """(state bytes, total bytes) of one decode step: the state is read once (M rows) and the K
    selected rows are written; inputs q, k, v, logits, f are read and o is written."""
    state = B * H * (M + K) * Dv * 4
    inputs = B * H * (2 * M * es + Dv * es + M * 4 + (M * 4 if per_slot else 4) + Dv * 4)
    return state, state + inputs


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples the SM clock and the throttle reasons every 10 ms (NVML, in a background thread;
    nvidia-smi at 200 ms if NVML is missing) while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int):
        import threading
        self.sm, self.smax, self.seen, self.err = [], None, set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self._phys_index(gpu_index))
            self.smax = float(pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM))
        except Exception as e:  # noqa: BLE001
            self._nv, self.err = None, f"nvml unavailable: {e}"
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()

    @staticmethod
    def _phys_index(i: int) -> int:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            try:
                return int(vis.split(",")[i])
            except (ValueError, IndexError):
                return i
        return i

    def _run(self):
        while not self._stop.is_set():
            if self._nv is not None:
                try:
                    self.sm.append(float(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM)))
                    r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                    for n, bit in self.REASONS.items():
                        if r & bit:
                            self.seen.add(n)
                except Exception as e:  # noqa: BLE001
                    self.err = str(e)
            self._stop.wait(0.01)

    def stop(self) -> dict:
        self._stop.set()
        self._t.join(timeout=2)
        out = {"sm_mhz": statistics.median(self.sm) if self.sm else None, "sm_max_mhz": self.smax,
               "samples": len(self.sm), "reasons": sorted(self.seen)}
        if self.err:
            out["note"] = self.err
        return out


# --------------------------------------------------------------------------- distributed

def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The maximum of `x` over all ranks (a device tensor under NCCL, a host tensor under gloo)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, ms_per_rank: float, world: int) -> tuple[float, float]:
    """Whole-job rate of N replicas: the units of all ranks over the slowest rank's time.
    Returns (rate per second, the max time in ms)."""
    ms_max = max_over_ranks(ms_per_rank, world)
    return units_per_rank * world / (ms_max * 1e-3), ms_max


def replica_seed(base: int, rank: int) -> int:
    """Each replica draws its own inputs."""
    return base + 1000 * rank


# --------------------------------------------------------------------------- CPU oracle timing

def pipelined_e2e(nsteps: int, warmup: int, h2d, compute, d2h, nsets: int = 2) -> float:
    """Mean ms per end-to-end step, device-timed, over `nsteps` steps run as a serving loop would:
    `nsets` device buffer sets and three streams, so the copies in of step i+1 and the read-back of
    step i overlap the computation. Every step still copies its own inputs in and its own result
    out inside the timed region. h2d(i, s), compute(i, s) and d2h(i, s) enqueue step i's work for
    buffer set s on the current stream."""
    import torch
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(nsets)]
    ev_comp = [torch.cuda.Event() for _ in range(nsets)]
    ev_out = [torch.cuda.Event() for _ in range(nsets)]

    def run(n, e0=None, e1=None):
        if e0 is not None:
            e0.record(s_in)
        for i in range(n):
            st = i % nsets
            with torch.cuda.stream(s_in):
                if i >= nsets:
                    s_in.wait_event(ev_comp[st])  # step i - nsets has consumed this set's inputs
                h2d(i, st)
                ev_in[st].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[st])
                if i >= nsets:
                    s_comp.wait_event(ev_out[st])  # step i - nsets's result has been read back
                compute(i, st)
                ev_comp[st].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[st])
                d2h(i, st)
                ev_out[st].record(s_out)
        if e1 is not None:
            e1.record(s_out)  # after the last read-back, which follows every earlier step's work
        torch.cuda.synchronize()

    run(max(1, warmup))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(nsteps, e0, e1)
    return e0.elapsed_time(e1) / nsteps


def oracle_sample(w, seconds_target: float = 3.0) -> dict:
    """Times the fp64 CPU oracle (as it stands) on a bounded sample of the workload: all heads of
    sequence 0, over a prefix of the tokens or, when the whole sequence is quick, repeated runs of
    it, for about `seconds_target` seconds of wall time on all host cores."""
    from oracle import oracle
    from sparse_routed_slot_b200.workloads import make_inputs

    cores = oracle.default_threads()

    def inputs(T):
        x = make_inputs(1, T, w.H, w.M, w.Dv, w.torch_dtype, w.decay, seed=w.seed)
        return {n: t.float().numpy() for n, t in x.items()}

    def run(c, reps=1):
        t0 = time.perf_counter()
        for _ in range(reps):
            oracle.forward(c["q"], c["k"], c["v"], c["logits"], c["f"], w.K, want_idx=False, nthreads=cores)
        return time.perf_counter() - t0

    T0 = min(w.T, 256)
    dt0 = run(inputs(T0))
    T1 = int(min(w.T, max(T0, T0 * seconds_target / max(dt0, 1e-6))))
    c1 = inputs(T1)
    dt1 = run(c1)
    reps = max(1, int(seconds_target / max(dt1, 1e-6))) if T1 == w.T else 1
    if reps > 1:
        dt1 = run(c1, reps)
    used = min(cores, w.H)
    return {"value": reps * T1 / dt1, "unit": "tokens/s", "cores": used, "kind": "oracle",
            "sample": f"sequence 0, all {w.H} heads, first {T1} of {w.T} tokens x {reps} run(s), fp64, "
                      f"{used} threads over heads; {dt1:.1f} s", "seconds": dt1, "tokens": T1 * reps}


def oracle_decode_sample(w, state, steps, state_bytes) -> dict:
    """Times the fp64 CPU oracle on the first steps of the generation workload, every stream,
    starting from the device's post-prefill state (upcast), and reports the state rate it reaches
    per step in the decode line's unit."""
    from oracle import oracle
    cores = oracle.default_threads()
    n = steps["q"].shape[0]
    t0 = time.perf_counter()
    for i in range(n):
        state = oracle.decode_step(steps["q"][i], steps["k"][i], steps["v"][i], steps["logits"][i], steps["f"][i],
                                   w.K, state, nthreads=cores)["state"]
    dt = (time.perf_counter() - t0) / n
    return {"value": state_bytes / dt / 1e9, "unit": "GB/s (state)", "cores": min(cores, w.B * w.H),
            "kind": "oracle", "ms_per_step": dt * 1e3,
            "sample": f"first {n} of {w.decode_steps} steps, all {w.B}x{w.H} streams, from the device's "
                      f"post-prefill state, fp64, {min(cores, w.B * w.H)} threads over streams"}


def _sources_digest() -> str:
    """sha256 of the CUDA sources (used to tell whether stored ncu counters are still current)."""
    from sparse_routed_slot_b200.profile_case import sources_digest
    return sources_digest()


def stored_tensor_pipe(kernel_prefix: str):
    """Tensor-pipe activity (% of elapsed cycles) of the first stored kernel whose name contains
    `kernel_prefix` (profiles/traffic.json, ncu section capture), or None when missing or stale."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(p))
    except (OSError, ValueError):
        return None
    if d.get("sources_sha256") != _sources_digest():
        return None
    for name, m in d.get("per_kernel", {}).items():
        if kernel_prefix in name and "tensor_pipe_pct" in m:
            return m["tensor_pipe_pct"]
    return None


def stored_traffic(key: str):
    """DRAM bytes per call measured by ncu for `key` (profiles/traffic.json), or None when the file
    is missing or was recorded for other kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(p))
    except (OSError, ValueError):
        return None
    if d.get("sources_sha256") != _sources_digest():
        return None
    return d.get("bytes", {}).get(key)


# --------------------------------------------------------------------------- our arm

KERNEL_NAMES = {4: ["route records", "segment summary", "segment scan", "chunk scan"],
                2: ["route records", "chunk scan"], 1: ["chunk scan (CUDA cores)"]}
L2_FLUSH_BYTES = 256 << 20  # written between timed steps of workloads smaller than L2 (126 MB)


class PrefillCase:
    """One prefill workload on the device: inputs, outputs, workspace and the timed call."""

    def __init__(self, w, dev, rank, path):
        import torch
        from sparse_routed_slot_b200 import api
        from sparse_routed_slot_b200.workloads import make_inputs
        self.w, self.path = w, path
        self.x = make_inputs(w.B, w.T, w.H, w.M, w.Dv, w.torch_dtype, w.decay,
                             seed=replica_seed(w.seed, rank), device=dev)
        self.o = torch.empty(w.B, w.T, w.H, w.Dv, dtype=torch.float32, device=dev)
        self.HT = torch.empty(w.B, w.H, w.M, w.Dv, dtype=torch.float32, device=dev)
        a = api._forward_args(self.x["q"], self.x["k"], self.x["v"], self.x["logits"], self.x["f"], w.K, None,
                              self.o, self.HT, None, None, path, False)
        self.path_used = api.selected_path(a)
        self.launches = api.kernel_launches(a)
        self.ws = torch.empty(max(api.workspace_bytes(a), 1), dtype=torch.uint8, device=dev)
        self.nbytes = prefill_bytes(w)
        self.flush = None if self.nbytes + o_fp32_extra_bytes(w) > L2_FLUSH_BYTES else \
            torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(self, x=None):
        import sparse_routed_slot_b200 as rsm
        x = self.x if x is None else x
        rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], self.w.K, out={"o": self.o, "HT": self.HT},
                    workspace=self.ws, path=self.path)

    def time(self, steps, warmup, world, stream, kernel_split=True):
        """Mean device time of one call (ms) and the per-kernel split (ms), CUDA events on the
        launching stream; the L2 is flushed between timed calls when the workload fits in it."""
        import ctypes
        import torch
        from sparse_routed_slot_b200 import _lib
        L = _lib.load()
        for _ in range(warmup):
            self.step()
        n = self.launches
        kev = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(steps)]
        for row in kev:  # torch creates the CUDA event on its first record
            for e in row:
                e.record(stream)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for a, b in ev:
            a.record(stream)
            b.record(stream)
        kev_ptrs = [(ctypes.c_void_p * (n + 1))(*[e.cuda_event for e in row]) for row in kev]
        torch.cuda.synchronize()
        barrier(world)
        for i in range(steps):
            if self.flush is not None:
                self.flush.zero_()
            if kernel_split:
                _lib.check(L.rsm_forward_set_profile_events(kev_ptrs[i], n + 1))
            ev[i][0].record(stream)
            self.step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        _lib.check(L.rsm_forward_set_profile_events(None, 0))
        barrier(world)
        ms = sum(a.elapsed_time(b) for a, b in ev) / steps
        kms = [sum(row[j].elapsed_time(row[j + 1]) for row in kev) / steps for j in range(n)] if kernel_split else []
        return ms, kms

    def time_graph(self, steps, warmup, world):
        """Mean device time of one call (ms) for workloads whose calls are shorter than the host's
        work to issue them: `steps` calls, each after an L2 flush, are captured in one CUDA graph
        and replayed; the time of a graph of the flushes alone is subtracted."""
        import torch
        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize()
        g_all, g_flush = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_all):
            for _ in range(steps):
                self.flush.zero_()
                self.step()
        with torch.cuda.graph(g_flush):
            for _ in range(steps):
                self.flush.zero_()
        stream = torch.cuda.current_stream()

        def replay(g, reps=5):
            g.replay()  # warm
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / reps

        barrier(world)
        t_all, t_flush = replay(g_all), replay(g_flush)
        barrier(world)
        del g_all, g_flush
        return max(t_all - t_flush, 1e-6) / steps

    def roofline(self, ms, peaks, traffic_key):
        achieved = self.nbytes / (ms * 1e-3) / 1e9
        w = self.w
        return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": stored_traffic(traffic_key),
                "algorithmic_bytes": self.nbytes, "o_fp32_extra_bytes": o_fp32_extra_bytes(w),
                "frac_with_o_fp32": (self.nbytes + o_fp32_extra_bytes(w)) / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "peak_source": peaks["source"] + " (burst copy)",
                "tensor_tflops": prefill_flops(w) / (ms * 1e-3) / 1e12,
                "chunk_scan_tensor_pipe_pct": stored_tensor_pipe("prefill_tc_kernel")
                if self.path_used == "tensor" else None}


def config_of(w, case, world, extra=None):
    c = {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "M": w.M, "K": w.K, "Dv": w.Dv,
         "decay": w.decay, "qkv_dtype": w.dtype, "state_dtype": "f32", "o_dtype": "f32",
         "path": case.path_used, "parallelism": f"replicas{world}",
         "l2": (f"L2 flushed between timed calls ({L2_FLUSH_BYTES >> 20} MB written)" if case.flush is not None
                else f"inputs larger than L2 ({case.nbytes / 1e6:.0f} MB per step, no flush)")}
    c.update(extra or {})
    return c


def run_ours(args, world, rank, local):
    import torch
    import sparse_routed_slot_b200 as rsm
    from sparse_routed_slot_b200.workloads import WORKLOADS

    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    stream = torch.cuda.current_stream(dev)
    case = PrefillCase(w, dev, rank, args.path)
    clocks = ClockSampler(local)
    ms, kms = case.time(args.steps, args.warmup, world, stream)
    clk = clocks.stop()
    names = KERNEL_NAMES.get(case.launches, [f"kernel {j}" for j in range(case.launches)])
    tokens = w.B * w.T
    value, ms_max = job_throughput(tokens, ms, world)

    # end to end through the public call with host buffers: every step copies its pinned inputs
    # in and reads o and H_T back, pipelined over two buffer sets (pipelined_e2e)
    import sparse_routed_slot_b200 as rsm
    host_in = {n: t.cpu().pin_memory() for n, t in case.x.items()}
    dev_in = [{n: torch.empty_like(t) for n, t in case.x.items()} for _ in range(2)]
    dev_out = [{"o": torch.empty_like(case.o), "HT": torch.empty_like(case.HT)} for _ in range(2)]
    wss = [torch.empty_like(case.ws) for _ in range(2)]
    host_out = [{"o": torch.empty(case.o.shape, dtype=case.o.dtype).pin_memory(),
                 "HT": torch.empty(case.HT.shape, dtype=case.HT.dtype).pin_memory()} for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = case.o.numel() * 4 + case.HT.numel() * 4

    def e2e_in(i, s):
        for n in host_in:
            dev_in[s][n].copy_(host_in[n], non_blocking=True)

    def e2e_compute(i, s):
        x = dev_in[s]
        rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], w.K, out=dev_out[s], workspace=wss[s],
                    path=case.path)

    def e2e_out(i, s):
        for n in ("o", "HT"):
            host_out[s][n].copy_(dev_out[s][n], non_blocking=True)

    barrier(world)
    e2e_ms = max_over_ranks(pipelined_e2e(args.steps, args.warmup, e2e_in, e2e_compute, e2e_out), world)
    del host_in, dev_in, dev_out, wss, host_out

    roof = case.roofline(ms, peaks, f"{w.name}/forward")
    roof["kernel"] = f"rsm_forward, all {case.launches} launches of the step (" + ", ".join(names) + ")"
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32" if case.path_used == "simt" else "tf32", "data": "synthetic",
        "config": config_of(w, case, world),
        "roofline": roof,
        "kernels": [{"name": n, "ms": t, "share": t / sum(kms) if sum(kms) > 0 else None}
                    for n, t in zip(names, kms)],
        "e2e": {"value": tokens * world / (e2e_ms * 1e-3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "pipelining": "two buffer sets, three streams: step i+1's copies in overlap step i"},
        "gpu_launches": 2 * args.steps * case.launches,  # device-timed steps and end-to-end steps
        "clocks": clk,
    }
    del case
    if rank == 0 and not args.no_cpu:
        line["cpu_baseline"] = oracle_sample(w)
    if not args.no_configs:
        line["configs"] = []
        for name in ("tiny_fp32", "small_bf16", "mid_gla_bf16"):
            sub = run_prefill_config(args, WORKLOADS[name], world, rank, local, peaks)
            line["gpu_launches"] += sub.pop("launches_timed")
            line["configs"].append(sub)
    if not args.no_configs:
        line["training"] = run_training(args, world, rank, local, peaks)
        line["gpu_launches"] += line["training"].pop("launches_timed")
    if not args.no_decode:
        line["decode"] = run_decode(args, world, rank, local, peaks)
        line["gpu_launches"] += line["decode"].pop("launches_timed")
    return line


def run_prefill_config(args, w, world, rank, local, peaks) -> dict:
    """A sub-line for another prefill workload: device time, roofline and the oracle beside it."""
    import torch
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    case = PrefillCase(w, dev, rank, args.path)
    steps = max(args.steps, 20)
    clocks = ClockSampler(local)
    ms, kms = case.time(steps, args.warmup, world, stream)
    timing = "CUDA events around each call on its stream"
    if case.flush is not None:
        # calls this small finish before the host has issued the next one: replay a captured graph
        ms = case.time_graph(steps, args.warmup, world)
        kms = []
        timing = (f"CUDA graph of {steps} calls, each after an L2 flush, replayed; a graph of the flushes "
                  f"alone subtracted")
    clk = clocks.stop()
    value, ms_max = job_throughput(w.B * w.T, ms, world)
    names = KERNEL_NAMES.get(case.launches, [f"kernel {j}" for j in range(case.launches)])
    roof = case.roofline(ms, peaks, f"{w.name}/forward")
    roof["kernel"] = f"rsm_forward, all {case.launches} launches of the step (" + ", ".join(names) + ")"
    sub = {"workload": w.name, "value": value, "unit": "tokens/s", "ms_per_step": ms_max, "steps": steps,
           "dtype": "f32" if case.path_used == "simt" else "tf32", "config": config_of(w, case, world),
           "roofline": roof,
           "kernels": [{"name": n, "ms": t} for n, t in zip(names, kms)], "clocks": clk, "timing": timing,
           "launches_timed": steps * case.launches * (1 if case.flush is None else 5)}
    if rank == 0 and not args.no_cpu:
        sub["cpu_baseline"] = oracle_sample(w)
    return sub


def backward_bytes(w) -> int:
    """Algorithmic bytes of one backward: the forward's inputs and dO read once, the gradients
    dq, dk, dlogits, dv, df and dH0 written once (fp32)."""
    es = 2 if w.dtype == "bf16" else 4
    th = w.B * w.T * w.H
    fsz = w.M * 4 if w.decay == "slot" else 4
    b = th * (2 * w.M * es + w.Dv * es + w.M * 4 + fsz + w.Dv * 4)   # q, k, v, logits, f, dO
    b += th * (3 * w.M * 4 + w.Dv * 4 + fsz)                         # dq, dk, dlogits, dv, df
    b += w.B * w.H * w.M * w.Dv * 4                                  # dH0
    return b


def run_training(args, world, rank, local, peaks) -> dict:
    """One training step of the mixer on the pages' small training shape: rsm_forward then
    rsm_backward, captured in a CUDA graph with an L2 flush before each step and replayed."""
    import torch
    import sparse_routed_slot_b200 as rsm
    from sparse_routed_slot_b200.workloads import WORKLOADS

    w = WORKLOADS["small_bf16"]
    dev = torch.device("cuda", local)
    case = PrefillCase(w, dev, rank, args.path)
    g = torch.Generator(device=dev).manual_seed(11 + rank)
    dO = torch.randn(w.B, w.T, w.H, w.Dv, generator=g, device=dev)
    grads = {"dq": torch.empty(w.B, w.T, w.H, w.M, device=dev), "dk": torch.empty(w.B, w.T, w.H, w.M, device=dev),
             "dlogits": torch.empty(w.B, w.T, w.H, w.M, device=dev), "dv": torch.empty(w.B, w.T, w.H, w.Dv, device=dev),
             "df": torch.empty(case.x["f"].shape, device=dev), "dH0": torch.empty(w.B, w.H, w.M, w.Dv, device=dev)}
    bws = torch.empty(1 << 24, dtype=torch.uint8, device=dev)
    x = case.x

    def bwd():
        rsm.backward(x["q"], x["k"], x["v"], x["logits"], x["f"], w.K, dO, None, None, out=grads, workspace=bws)

    fwd_step = case.step

    def step():
        fwd_step()
        bwd()

    case.step = step
    steps = max(args.steps, 20)
    clocks = ClockSampler(local)
    ms_train = case.time_graph(steps, args.warmup, world)
    case.step = bwd
    ms_bwd = case.time_graph(steps, args.warmup, world)
    clk = clocks.stop()
    nb = backward_bytes(w)
    value, ms_max = job_throughput(w.B * w.T, ms_train, world)
    return {"workload": w.name, "value": value, "unit": "tokens/s (forward + backward)", "ms_per_step": ms_max,
            "ms_backward": ms_bwd, "steps": steps, "dtype": "f32 (backward on CUDA cores)",
            "roofline": {"bound": "hbm", "achieved": nb / (ms_bwd * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": nb / (ms_bwd * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "algorithmic_bytes": nb, "kernel": "rsm_backward (routing + one sweep kernel)",
                         "peak_source": peaks["source"] + " (burst copy)"},
            "timing": f"CUDA graph of {steps} steps, each after an L2 flush, replayed; flushes subtracted",
            "context": "the pages' only speed figure is whole-model training of a 35M-parameter model on an "
                       "RTX 4090 (about 49.6K tokens/s); not comparable with one mixer layer",
            "clocks": clk, "launches_timed": steps * (case.launches + 2) * 5 + steps * 2 * 5}


def run_decode(args, world, rank, local, peaks) -> dict:
    """Generation decode: 256 sequences x 16 heads, state from a 2048-token prefill, then every
    step of the workload (1024 rsm_decode_step calls, one launch each) timed on the device."""
    import torch
    import sparse_routed_slot_b200 as rsm
    from sparse_routed_slot_b200.workloads import DECODE_PREFILL_GROUP, WORKLOADS, decode_prefill_group, \
        decode_step_inputs

    w = WORKLOADS["decode_256x16"]
    dev = torch.device("cuda", local)
    state = torch.zeros(w.B, w.H, w.M, w.Dv, dtype=torch.float32, device=dev)
    for b0 in range(0, w.B, DECODE_PREFILL_GROUP):
        x = decode_prefill_group(w, b0, rank, device=dev)
        out = rsm.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], w.K, state=True, path=args.path)
        state[b0:b0 + DECODE_PREFILL_GROUP].copy_(out["HT"])
        del x, out
    state0 = state.clone() if rank == 0 and not args.no_cpu else None
    nsteps = args.decode_steps
    d = decode_step_inputs(w, nsteps, rank, device=dev)
    o = torch.empty(w.B, w.H, w.Dv, dtype=torch.float32, device=dev)

    def step(i, x=d):
        rsm.decode_step(x["q"][i], x["k"][i], x["v"][i], x["logits"][i], x["f"][i], w.K, state, o=o)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    stream = torch.cuda.current_stream(dev)
    clocks = ClockSampler(local)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(nsteps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / nsteps, world)
    sb, tb = decode_bytes(w.B, w.H, w.M, w.K, w.Dv, 2, w.decay == "slot")
    state_gbs = sb / (ms * 1e-3) / 1e9
    total_gbs = tb / (ms * 1e-3) / 1e9

    # end to end: every step's inputs copied in from pinned host memory and o read back; the
    # carried state stays on the device (it is the recurrence's own memory)
    e2e_steps = min(nsteps, 256)
    host_in = {n: t[:e2e_steps].cpu().pin_memory() for n, t in d.items()}
    dev_in = [{n: torch.empty_like(t[0]) for n, t in d.items()} for _ in range(2)]
    dev_o = [torch.empty_like(o) for _ in range(2)]
    host_o = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t[0].numel() * t.element_size() for t in host_in.values())

    def e2e_in(i, s):
        for n in host_in:
            dev_in[s][n].copy_(host_in[n][i % e2e_steps], non_blocking=True)

    def e2e_compute(i, s):  # the steps stay in order on one stream: the state carries between them
        x = dev_in[s]
        rsm.decode_step(x["q"], x["k"], x["v"], x["logits"], x["f"], w.K, state, o=dev_o[s])

    def e2e_out(i, s):
        host_o[s].copy_(dev_o[s], non_blocking=True)

    barrier(world)
    e2e_ms = max_over_ranks(pipelined_e2e(e2e_steps, 3, e2e_in, e2e_compute, e2e_out), world)
    cpu_steps = {n: t[:8].float().cpu().numpy() for n, t in d.items()} if state0 is not None else None
    del host_in, dev_in, d

    res = {"value": state_gbs * world, "unit": "GB/s (state, all GPUs)", "ms_per_step": ms,
           "steps_timed": nsteps, "total_gbs": total_gbs * world,
           "tokens_per_s": w.B * world / (ms * 1e-3),
           "roofline": {"bound": "hbm", "achieved": total_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": total_gbs / peaks["hbm_gbs"],
                        "traffic": stored_traffic("decode_256x16/step"),
                        "algorithmic_bytes": tb, "kernel": "rsm_decode_step (one launch per step)",
                        "peak_source": peaks["source"] + " (burst copy)"},
           "e2e": {"value": sb * world / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s (state, all GPUs)",
                   "ms_per_step": e2e_ms, "steps": e2e_steps,
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": o.numel() * 4,
                   "pipelining": "two buffer sets, three streams: step i+1's copies in overlap step i"},
           "clocks": clk, "launches_timed": nsteps + e2e_steps,
           "config": {"workload": w.name, "B": w.B, "H": w.H, "M": w.M, "K": w.K, "Dv": w.Dv,
                      "decay": w.decay, "qkv_dtype": w.dtype, "prefill_T": w.decode_prefill_T,
                      "graph": False, "l2": f"state {w.B * w.H * w.M * w.Dv * 4 / 1e6:.0f} MB > L2, no flush"}}
    if state0 is not None:
        res["cpu_baseline"] = oracle_decode_sample(w, state0.double().cpu().numpy(), cpu_steps, sb)
    return res


# --------------------------------------------------------------------------- reference arm

def run_reference(args, world, rank) -> dict | None:
    from sparse_routed_slot_b200.workloads import WORKLOADS
    if rank != 0:
        return None
    w = WORKLOADS[args.workload]
    for _ in range(args.warmup):
        oracle_sample(w, seconds_target=2.0)
    vals, secs = [], 0.0
    last = None
    for _ in range(args.steps):
        last = oracle_sample(w, seconds_target=6.0)
        vals.append(last["value"])
        secs += last["seconds"]
    value = sum(vals) / len(vals)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * last["tokens"] / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "M": w.M, "K": w.K, "Dv": w.Dv,
                       "decay": w.decay, "qkv_dtype": w.dtype},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": last["cores"], "kind": "oracle",
                             "sample": last["sample"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_ctx_bf16")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "tensor"])
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-configs", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    world, rank, local = dist_setup()
    line = run_ours(args, world, rank, local)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
