"""The bench's N>1 host logic on CPU: two gloo ranks, max-over-ranks timing and the
whole-job throughput (replicas only: each rank decodes its own batch, no data-path
collective)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    import datetime

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [12.5, 20.0][rank]  # rank 1 is the slow one
        max_ms = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        value = bench.job_throughput(world, 64, 512, 1000, max_ms)
        out[rank] = (max_ms, value)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    # every rank sees the slowest rank's time; throughput counts all ranks' work over it
    for r in range(world):
        max_ms, value = out[r]
        assert max_ms == pytest.approx(20.0)
        assert value == pytest.approx(2 * 64 * 512 * 1000 / 20e-3)


def test_single_rank_helpers_without_a_process_group():
    import bench

    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.job_throughput(1, 64, 512, 10, 1.0) == pytest.approx(64 * 512 * 10 / 1e-3)
