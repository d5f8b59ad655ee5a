"""The N-GPU benchmark runs independent replicas (the path shards by sequence and head with no
exchange): the whole-job rate is all ranks' units over the slowest rank's time. These checks run
the host side of that with two gloo ranks on CPU (no GPU, no collective on a data path)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = [2.0, 3.5][rank]  # rank 1 is the slowest
        rate, ms_max = bench.job_throughput(1000, ms, world)
        seed = bench.replica_seed(3, rank)
        bench.barrier(world)
        q.put((rank, rate, ms_max, seed))
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, rate, ms_max, seed in res:
        assert ms_max == pytest.approx(3.5)                 # max over ranks, on every rank
        assert rate == pytest.approx(2 * 1000 / 3.5e-3)     # all units over the slowest time
    assert res[0][3] != res[1][3]                           # each replica has its own inputs


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    rate, ms_max = bench.job_throughput(500, 4.0, 1)
    assert ms_max == 4.0 and rate == pytest.approx(500 / 4e-3)
