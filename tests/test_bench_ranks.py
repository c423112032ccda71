"""Host logic of the multi-rank bench path (one process per GPU, timing taken
as the max over ranks, whole-job throughput), run as two gloo ranks on CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 19.0][rank]                       # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, torch.device("cpu"), world)
        rate = bench.whole_job_rate(1.0e12, world, ms_max)
        q.put((rank, ms_max, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms_max, rate in got:
        assert ms_max == 19.0                         # every rank sees the slowest time
        assert rate == pytest.approx(2 * 1.0e12 / 19.0e-3)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.25, torch.device("cpu"), 1) == 3.25
    assert bench.whole_job_rate(6.0e12, 1, 2.0) == pytest.approx(3.0e15)
