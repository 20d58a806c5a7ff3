"""The multi-process plumbing of bench.py on CPU ranks (gloo, world size 2):
the slowest rank's time is what every rank reports, and the whole-job value
counts the units of all ranks (independent replicas, no data-path
collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms = 1.5 * (rank + 1)                      # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, world)
        value = bench.aggregate_throughput(8192, world, ms_max)
        results[rank] = (ms_max, value)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert results[0] == results[1]
    ms_max, value = results[0]
    assert ms_max == pytest.approx(3.0)
    assert value == pytest.approx(2 * 8192 / 3.0e-3)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(2.5, 1) == 2.5
    assert bench.aggregate_throughput(64, 1, 0.5) == pytest.approx(128000.0)
