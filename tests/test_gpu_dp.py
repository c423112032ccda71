"""fp4_allreduce_sum_f32, the data-parallel dW sum behind the C ABI, on the
GPU: with a one-rank NCCL communicator (every call in this environment has
one GPU) the sum over the ranks is the buffer itself; the call is enqueued on
the given stream after the work queued there.  The multi-rank ordering of
the sums in the step is tested on CPU ranks (test_bench_ranks.py)."""
import pytest
import torch

import bench

pytestmark = pytest.mark.gpu


def test_allreduce_one_rank_is_identity_and_stream_ordered(gpu_lib):
    F = gpu_lib
    comm = F.NcclComm(0, 1)
    try:
        s = torch.cuda.Stream()
        buf = torch.zeros(3 * 1024 + 5, dtype=torch.float32, device="cuda")
        with torch.cuda.stream(s):
            buf.copy_(torch.arange(buf.numel(), dtype=torch.float32, device="cuda") * 0.5)
            F.fp4_allreduce_sum_f32(comm, buf, stream=s)
            out = buf.clone()
        torch.cuda.synchronize()
        assert torch.equal(out, torch.arange(buf.numel(), dtype=torch.float32, device="cuda") * 0.5)
        dp = bench.DwAllReduce(2, F, comm)        # the step's orchestration on the library path
        dw = torch.full((256, 64), 3.0, dtype=torch.float32, device="cuda")
        dp.issue(dw)
        dp.finish()
        torch.cuda.synchronize()
        assert (dw == 3.0).all()
    finally:
        comm.destroy()
