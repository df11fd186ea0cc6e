"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

Rows are independent, so N GPUs run N replicas of the workload with no
collective on the data path; the only cross-rank step is taking the slowest
rank's time.  These tests run that step with two gloo ranks on 127.0.0.1.
"""
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


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        mine = 10.0 + 5.0 * rank          # rank 1 is the slow one
        got = bench.max_over_ranks(mine, dist, torch.device("cpu"))
        value = bench.job_gbs(1e9, 4, world, got)
        out.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_slowest_rank_sets_the_time_and_value_counts_all_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, got, value in res:
        assert got == 15.0                       # max over ranks, on every rank
        assert value == pytest.approx(1e9 * 4 * 2 / 0.015 / 1e9)


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(3.5, dist, torch.device("cpu")) == 3.5
    assert bench.job_gbs(2e9, 10, 1, 1000.0) == pytest.approx(20.0)
