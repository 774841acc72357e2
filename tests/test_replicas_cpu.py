"""The replica path of bench.py (N > 1: one independent replica per GPU, no
data-path collective) on CPU: two gloo ranks agree on the slowest rank's time
and on the whole-job throughput."""
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


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = 1.0 + rank          # rank 1 is the slow replica
        slowest = bench.replica_max(elapsed, dist, torch.device("cpu"))
        out[rank] = (slowest, bench.job_rate(1000.0, 10, world, slowest))
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(world):
        slowest, rate = res[r]
        assert slowest == 2.0
        assert rate == pytest.approx(1000.0 * 10 * 2 / 2.0)


def test_single_process_needs_no_group():
    assert bench.replica_max(3.5) == 3.5
    assert bench.job_rate(8.0, 4, 1, 2.0) == 16.0
