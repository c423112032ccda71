"""fp4_gemm_noalloc: the GEMM entry point for callers that cannot allocate
device memory (code running while a framework's pool owns every device
allocation, plugins in processes that forbid it, paths that must not risk the
synchronisation cudaMalloc can cause).  Its scratch is a static array held by
the library on each device.

Collected last on purpose: if it fails, a run that stops at the first
failure has already run every other test.  It must pass both alone in a
fresh process and after the other tests (the array then holds the previous
calls' contents)."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import fqt_synth as S
import oracle as O
from conftest import ROOT
from fp4_testlib import rel_fro, upload_qtensor

pytestmark = pytest.mark.gpu
TOL = 1e-3


def _pair(F, M, N, K, seed):
    a, b = S.sparse_outliers(M, K, seed=seed), S.normal((N, K), 0.02, seed=seed + 1)
    qa = O.nvfp4_quantize_1d(S.as_f32(a))
    qb = O.nvfp4_quantize_2d(S.as_f32(b))
    ref = O.gemm(O.dequantize(qa["codes"], qa["scales"]),
                 O.dequantize(qb["codes"], qb["scales"], (16, 16)), alpha=0.5,
                 s_dec_a=qa["s_dec"], s_dec_b=qb["s_dec"])
    return upload_qtensor(F, qa, M, K, 0, 0), upload_qtensor(F, qb, N, K, 0, 1), ref


@pytest.mark.parametrize("M,N,K,seed", [(256, 384, 512, 1), (128, 256, 320, 2)])
def test_noalloc_gemm_matches_fp4_gemm_on_two_calls(gpu_lib, M, N, K, seed):
    """Two calls in a row: each bit for bit equal to fp4_gemm on the same
    operands (the same kernel runs), within 1e-3 of the float64 oracle, and
    with the output amax of its own result."""
    F = gpu_lib
    ta, tb, ref = _pair(F, M, N, K, seed)
    want = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    ws = F.Workspace(M, N, K)
    F.fp4_gemm(ta, tb, want, alpha=0.5, ws=ws)
    for _ in range(2):
        amax = torch.zeros(1, dtype=torch.float32, device="cuda")
        got = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        F.fp4_gemm_noalloc(ta, tb, got, alpha=0.5, c_amax=amax)
        torch.cuda.synchronize()
        assert ws.status() == 0
        assert torch.equal(got, want)
        g = got.cpu().numpy()
        assert rel_fro(g, ref) <= TOL
        assert float(amax.item()) == float(np.abs(g).max())


def test_noalloc_gemm_rejects_bad_arguments(gpu_lib):
    F = gpu_lib
    ta, tb, _ = _pair(F, 128, 256, 256, 3)
    out = torch.zeros((128, 200), dtype=torch.float32, device="cuda")
    with pytest.raises(F.Fp4Error) as e:
        F.fp4_gemm_noalloc(ta, tb, out[:, :200])       # N mismatch / leading dimension
    assert e.value.code in (2, 3)


_RETRY_CHILD = r"""
import sys, torch
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
import fp4_fully_quantized_b200 as F
from test_zz_no_alloc import _pair
ta, tb, _ = _pair(F, 128, 256, 256, 4)
want = torch.zeros((128, 256), dtype=torch.float32, device="cuda")
F.fp4_gemm(ta, tb, want, alpha=0.5)
got = torch.zeros_like(want)
try:
    F.fp4_gemm_noalloc(ta, tb, got, alpha=0.5)
    print("first call did not fail"); sys.exit(1)
except F.Fp4Error as e:
    assert e.code == 6, e.code                      # FP4_ERR_CUDA, nothing enqueued
F.fp4_gemm_noalloc(ta, tb, got, alpha=0.5)
torch.cuda.synchronize()
assert torch.equal(got, want)
print("retry ok")
"""


def test_noalloc_lookup_failure_is_not_kept(gpu_lib):
    """A failed look-up of the scratch array's device address (simulated on
    the host for the first look-up of a fresh process) returns FP4_ERR_CUDA,
    and the next call looks it up again and computes the product."""
    env = dict(os.environ, FP4_NOALLOC_FAIL_LOOKUPS="1", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", _RETRY_CHILD, ROOT], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and "retry ok" in r.stdout, r.stdout + r.stderr
