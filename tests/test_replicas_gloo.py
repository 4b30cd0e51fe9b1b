"""The multi-GPU path is replicas only (the layer has no data-path exchange):
every rank runs its own copy of the step and the bench reports the slowest
rank's time, with whole-job throughput = all ranks' work / that time.  The
host-side logic of that path runs here on CPU with two gloo ranks."""
import multiprocessing as mp
import os
import socket

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r "measured" (10 + r) ms for the timed steps and (30 - r) ms end to end
        got = bench.max_over_ranks([10.0 + rank, 30.0 - rank], "cpu")
        value = bench.job_throughput(2.0e9, 5, world, got[0])
        q.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, value in res:
        assert got == [11.0, 30.0]                      # slowest rank, per quantity
        assert value == pytest.approx(2.0e9 * 5 * 2 / 11.0e-3)


def test_single_process_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5], "cpu") == [1.5, 2.5]
    assert bench.job_throughput(1.0e9, 10, 1, 5.0) == pytest.approx(2.0e12)
