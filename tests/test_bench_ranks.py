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


def _dp_rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dp = bench.DwAllReduce(world)
        # two layers' dW, distinct per rank; sums issued in layer order, joined at the end
        dws = [torch.full((4, 8), float(rank + 1)), torch.arange(12.0).reshape(3, 4) * (rank + 1)]
        for dw in dws:
            dp.issue(dw)
        assert len(dp.works) == 2
        dp.finish()
        assert dp.works == []
        q.put((rank, dws[0].tolist(), dws[1].tolist()))   # plain lists: tensors would be shared by fd
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_dw_allreduce_gloo_two_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_dp_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted((q.get(timeout=5) for _ in range(world)), key=lambda t: t[0])
    for _rank, a, b in got:
        assert torch.equal(torch.tensor(a), torch.full((4, 8), 3.0))          # 1 + 2
        assert torch.equal(torch.tensor(b), torch.arange(12.0).reshape(3, 4) * 3)


def test_dw_allreduce_single_rank_is_a_no_op():
    dp = bench.DwAllReduce(1)
    dw = torch.ones(2, 2)
    dp.issue(dw)
    dp.finish()
    assert dp.works == [] and torch.equal(dw, torch.ones(2, 2))


def test_plan_places_the_dw_sum_after_each_wgrad():
    from types import SimpleNamespace as NS
    cfg = NS(fmt=0, rht_n=0, rht_mask=0, round_fwd=0, round_x_t=1, round_bwd=1, seed=0, w_block=1)
    layers = [NS(name=f"l{i}", N=256, K=128, M=512, cfg=cfg, sv=NS(), dw=None) for i in range(3)]
    labels = [c[3] for c in bench.plan(None, layers, ws=None, dp=bench.DwAllReduce(2))]
    kinds = [c[0] for c in bench.plan(None, layers, ws=None, dp=bench.DwAllReduce(2))]
    assert len(labels) == 3 * 7 + 1 and labels[-1] == "dW all-reduce wait"
    for i in range(3):
        assert labels[7 * i + 5].startswith("wgrad l%d" % i)
        assert labels[7 * i + 6].startswith("dW all-reduce l%d" % i)
    assert kinds.count("comm") == 4
    assert [c[3] for c in bench.plan(None, layers, ws=None)][-1].startswith("wgrad l2")
