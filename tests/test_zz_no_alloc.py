"""fp4_gemm_noalloc: the GEMM entry point for callers that cannot allocate
device memory (its scratch is a static array held by the library).

Collected last on purpose: if it fails, a run that stops at the first
failure has already run every other test.  It must pass both alone in a
fresh process and after the other tests (the array then holds the previous
calls' contents)."""
import numpy as np
import pytest
import torch

import fqt_synth as S
import oracle as O
from fp4_testlib import rel_fro, upload_qtensor

pytestmark = pytest.mark.gpu
TOL = 1e-3


def _pair(F, M, N, K, seed):
    a, b = S.sparse_outliers(M, K, seed=seed), S.normal((N, K), 0.02, seed=seed + 1)
    qa = O.nvfp4_quantize_1d(S.as_f32(a))
    qb = O.nvfp4_quantize_2d(S.as_f32(b))
    return upload_qtensor(F, qa, M, K, 0, 0), upload_qtensor(F, qb, N, K, 0, 1)


def test_noalloc_gemm_matches_fp4_gemm_on_two_calls(gpu_lib):
    F = gpu_lib
    for M, N, K, seed in ((256, 384, 512, 1), (128, 256, 320, 2)):
        ta, tb = _pair(F, M, N, K, seed)
        ref = torch.zeros((M, N), dtype=torch.float32, device="cuda")
        ws = F.Workspace(M, N, K)
        F.fp4_gemm(ta, tb, ref, alpha=0.5, ws=ws)
        amax = torch.zeros(1, dtype=torch.float32, device="cuda")
        got = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        F.fp4_gemm_noalloc(ta, tb, got, alpha=0.5, c_amax=amax)
        torch.cuda.synchronize()
        assert ws.status() == 0
        g, r = got.cpu().numpy(), ref.cpu().numpy()
        assert np.isfinite(g).all()
        assert rel_fro(g, r) <= TOL
        assert float(amax.item()) == float(np.abs(g).max())


def test_noalloc_gemm_rejects_bad_arguments(gpu_lib):
    F = gpu_lib
    ta, tb = _pair(F, 128, 256, 256, 3)
    out = torch.zeros((128, 200), dtype=torch.float32, device="cuda")
    with pytest.raises(F.Fp4Error) as e:
        F.fp4_gemm_noalloc(ta, tb, out[:, :200])       # N mismatch / leading dimension
    assert e.value.code in (2, 3)
