"""Chained SwiGLU MLP stack (8 layers, hidden 2048, FFN 8192, 16384 tokens):
NVFP4 forward through every layer, SR gradients back, each linear through
fqt_linear_fwd / fqt_linear_bwd.  Checks: sampled rows of the first and last
layers' quantized operands are bit-exact with the oracle; every error against
the unquantized FP32 stack is finite; the first layer's activations carry
NVFP4-sized noise (a relative error of at most 0.3: E2M1 round-to-nearest is
off by at most a quarter of a value above the block's smallest level, and the
GEMM averages that over the contraction); no layer diverges (all < 2)."""
import math

import pytest
import torch

import bench

pytestmark = pytest.mark.gpu


def _check(res):
    assert res["oracle_rows_checked"] > 0
    assert res["oracle_mismatches"] == 0
    rows = res["rel_err_vs_fp32"]
    for r in rows:
        for k in ("act", "dx", "dw_gate_up", "dw_down"):
            assert math.isfinite(r[k]), (r, k)
            assert r[k] < 2.0, (r, k)
    assert rows[0]["act"] < 0.3


def test_swiglu_stack_small(gpu_lib):
    res = bench.run_swiglu(torch.device("cuda", 0), layers=3, hidden=256, ffn=512, tokens=1024)
    _check(res)


def test_swiglu_stack_full_config(gpu_lib):
    res = bench.run_swiglu(torch.device("cuda", 0))
    print(res)
    _check(res)
