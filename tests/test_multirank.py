"""Multi-rank host logic of the benchmark, on CPU with gloo (world size 2).

The layer step has no exchange between GPUs: each rank runs an independent
replica. What must be right across ranks is the aggregation: the slowest
rank's time, and the units of all ranks.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dev = torch.device("cpu")
        # rank r took (10 + 5r) ms for (100 + r) rows
        ms, units, value = bench.aggregate(10.0 + 5.0 * rank, 100.0 + rank, dev)
        bench.barrier()
        q.put((rank, ms, units, value))
    finally:
        dist.destroy_process_group()


def test_aggregate_two_ranks_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0, f"rank process exited with {p.exitcode}"
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, units, value in res:
        assert ms == pytest.approx(15.0)          # max over ranks
        assert units == pytest.approx(201.0)      # sum over ranks
        assert value == pytest.approx(201.0 / 0.015)


def test_aggregate_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    ms, units, value = bench.aggregate(20.0, 64.0, "cpu")
    assert (ms, units) == (20.0, 64.0)
    assert value == pytest.approx(3200.0)
