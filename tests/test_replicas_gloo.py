"""The N > 1 path of bench.py on the CPU: world_size-2 gloo ranks, each a replica of the decode
step, agree on barriers and take the maximum of their times (the slowest rank sets the clock), and
the whole-job throughput counts every rank's units. No GPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.rank_barrier(dist)
        ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
        out[rank] = (bench.max_over(dist, ms, "cpu"), bench.replica_throughput(world, 100, bench.max_over(dist, ms, "cpu")))
        bench.rank_barrier(dist)
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_max_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert out[0] == out[1] == (15.0, world * 100 / 0.015)


def test_single_rank_helpers_are_identity():
    import bench
    bench.rank_barrier(None)
    assert bench.max_over(None, 3.5, "cpu") == 3.5
    assert bench.replica_throughput(1, 10, 2.0) == pytest.approx(5000.0)
