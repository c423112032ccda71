"""Config 4: MXFP4 against NVFP4 on the same seeded Llama-7B-shaped
tensors ("FP4" page, Components, NVFP4: lower quantization error than
MXFP4).  Trend checks only: per operand, rounded to nearest in both formats,
NVFP4's relative quantization noise is below MXFP4's; the forward product
(round to nearest in both layer configurations) is closer to the unquantized
float64 product in NVFP4; every product carries an FP4-sized error.  (The
NVFP4 layer's stochastically rounded gradients are noisier than MXFP4's
round-to-nearest ones by design, so its dX and dW are not compared.)"""
import pytest
import torch

import bench

pytestmark = pytest.mark.gpu


def test_nvfp4_quantization_noise_below_mxfp4(gpu_lib):
    res = bench.run_formats(torch.device("cuda", 0), rows_checked=32, M=4096)
    for row in res["shapes"]:
        nv, mx = row["noise"]["nvfp4"], row["noise"]["mxfp4"]
        for op in ("X", "W", "dY"):
            assert 0.0 < nv[op] < mx[op], (row["layer"], op, nv[op], mx[op])
        assert row["gemm_err"]["nvfp4"]["Y"] < row["gemm_err"]["mxfp4"]["Y"]
        for fmt in ("nvfp4", "mxfp4"):
            for prod, err in row["gemm_err"][fmt].items():
                assert 0.0 < err < 0.35, (row["layer"], fmt, prod, err)
