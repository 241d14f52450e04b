"""Host logic of the multi-GPU benchmark on CPU: two gloo ranks, each with its own
step time, agree on the slowest rank's time, and the job throughput counts every
rank's tokens over that time (weak scaling: one sequence per rank)."""
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


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [7.5, 9.25][rank]
        ms_max = bench.max_over_ranks(ms, world, torch.device("cpu"))
        q.put((rank, ms_max, bench.job_throughput(10240, world, 3, ms_max)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[1] for g in got] == [9.25, 9.25]
    assert got[0][2] == pytest.approx(2 * 10240 * 3 / 9.25e-3)


def test_single_rank_needs_no_collective():
    assert bench.max_over_ranks(3.0, 1, torch.device("cpu")) == 3.0
    assert bench.job_throughput(100, 1, 2, 1000.0) == pytest.approx(200.0)
