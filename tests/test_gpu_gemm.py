"""tcgen05 block-scaled FP4 GEMM vs the oracle's float64 GEMM.

Both sides multiply the SAME quantized operands: they are produced by the
oracle quantizer on the CPU and uploaded, so this isolates the GEMM.  The
bar is a relative Frobenius error <= 1e-3 on FP32 outputs (the tensor cores
accumulate in FP32; the oracle sums exactly in float64).
"""
import numpy as np
import pytest
import torch

import fqt_synth as S
import oracle as O
from fp4_testlib import rel_fro, upload_qtensor

pytestmark = pytest.mark.gpu
TOL = 1e-3


def _operands(F, M, N, K, fmt, seed=0, w_2d=False):
    a = S.sparse_outliers(M, K, seed=seed)
    b = S.normal((N, K), 0.02, seed=seed + 1)
    af, bf = S.as_f32(a), S.as_f32(b)
    if fmt == 0:
        qa = O.nvfp4_quantize_1d(af)
        qb = O.nvfp4_quantize_2d(bf) if w_2d else O.nvfp4_quantize_1d(bf)
        blk_b = (16, 16) if w_2d else (1, 16)
        ah = O.dequantize(qa["codes"], qa["scales"])
        bh = O.dequantize(qb["codes"], qb["scales"], block=blk_b)
    else:
        qa, qb = O.mxfp4_quantize(af), O.mxfp4_quantize(bf)
        ah = O.dequantize(qa["codes"], qa["scales"], (1, 32), True)
        bh = O.dequantize(qb["codes"], qb["scales"], (1, 32), True)
    ta = upload_qtensor(F, qa, M, K, fmt, 0)
    tb = upload_qtensor(F, qb, N, K, fmt, 1 if w_2d else 0)
    return ta, tb, ah, bh, qa, qb


SHAPES = [(128, 256, 256), (128, 128, 64), (256, 384, 320), (384, 512, 1024), (128, 256, 128),
          (256, 128, 192)]


@pytest.mark.parametrize("mnk", SHAPES)
def test_gemm_nvfp4_small_shapes(gpu_lib, mnk):
    _small(gpu_lib, 0, mnk)


def _small(F, fmt, mnk):
    M, N, K = mnk
    ta, tb, ah, bh, qa, qb = _operands(F, M, N, K, fmt, seed=M + N + K)
    out = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    ws = F.Workspace(M, N, K)
    F.fp4_gemm(ta, tb, out, alpha=1.5, c_amax=amax, ws=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    ref = O.gemm(ah, bh, alpha=1.5, s_dec_a=qa["s_dec"], s_dec_b=qb["s_dec"])
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    err = rel_fro(got, ref)
    assert err <= TOL, err
    assert abs(float(amax.item()) - np.abs(got).max()) <= 1e-6 * np.abs(got).max()


def test_gemm_bf16_output_and_2d_weights(gpu_lib):
    F = gpu_lib
    M, N, K = 256, 512, 512
    ta, tb, ah, bh, qa, qb = _operands(F, M, N, K, 0, seed=3, w_2d=True)
    out = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    F.fp4_gemm(ta, tb, out)
    torch.cuda.synchronize()
    ref = O.gemm(ah, bh, s_dec_a=qa["s_dec"], s_dec_b=qb["s_dec"])
    got = out.float().cpu().numpy()
    # BF16 rounding of the output alone is ~2^-9 relative per element
    assert rel_fro(got, ref) <= 4e-3
    # and the unrounded FP32 path agrees with the oracle to 1e-3
    out32 = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    F.fp4_gemm(ta, tb, out32)
    torch.cuda.synchronize()
    assert rel_fro(out32.cpu().numpy(), ref) <= TOL
    assert torch.equal(out.cpu(), out32.to(torch.bfloat16).cpu())


def test_gemm_leading_dimension(gpu_lib):
    F = gpu_lib
    M, N, K = 128, 256, 256
    ta, tb, ah, bh, qa, qb = _operands(F, M, N, K, 0, seed=8)
    big = torch.full((M, N + 64), 7.0, dtype=torch.float32, device="cuda")
    F.fp4_gemm(ta, tb, big[:, :N])
    torch.cuda.synchronize()
    ref = O.gemm(ah, bh, s_dec_a=qa["s_dec"], s_dec_b=qb["s_dec"])
    assert rel_fro(big[:, :N].cpu().numpy(), ref) <= TOL
    assert (big[:, N:] == 7.0).all()


def test_gemm_zero_and_one_hot(gpu_lib):
    F = gpu_lib
    M, N, K = 128, 128, 128
    A = np.zeros((M, K), np.float32)
    A[np.arange(M), np.arange(M) % K] = 4.0
    B = S.as_f32(S.normal((N, K), 1.0, seed=2))
    qa, qb = O.nvfp4_quantize_1d(A), O.nvfp4_quantize_1d(B)
    ta, tb = upload_qtensor(F, qa, M, K, 0, 0), upload_qtensor(F, qb, N, K, 0, 0)
    out = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    F.fp4_gemm(ta, tb, out)
    torch.cuda.synchronize()
    ref = O.gemm(O.dequantize(qa["codes"], qa["scales"]), O.dequantize(qb["codes"], qb["scales"]),
                 s_dec_a=qa["s_dec"], s_dec_b=qb["s_dec"])
    assert rel_fro(out.cpu().numpy(), ref) <= 1e-6
    Z = np.zeros((M, K), np.float32)
    qz = O.nvfp4_quantize_1d(Z)
    tz = upload_qtensor(F, qz, M, K, 0, 0)
    F.fp4_gemm(tz, tb, out)
    torch.cuda.synchronize()
    assert (out == 0).all()


@pytest.mark.parametrize("nk", [(11008, 4096), (4096, 11008)])
def test_gemm_llama_fprop_sampled_rows(gpu_lib, nk):
    """7B-shape fprop at full size (M = 32768) in the bench's launch
    configuration; 128 sampled output rows are checked against the float64
    oracle over the full contraction."""
    F = gpu_lib
    N, K = nk
    M = 32768
    d = S.llama_linear(N, K, M=M, seed=0)
    xf, wf = S.as_f32(d["X"]), S.as_f32(d["W"])
    qx = O.nvfp4_quantize_1d(xf)
    qw = O.nvfp4_quantize_2d(wf)
    ta = upload_qtensor(F, qx, M, K, 0, 0)
    tb = upload_qtensor(F, qw, N, K, 0, 1)
    out = torch.empty((M, N), dtype=torch.float32, device="cuda")
    ws = F.Workspace(M, N, K)
    F.fp4_gemm(ta, tb, out, ws=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    rows = np.sort(np.random.default_rng(5).choice(M, 128, replace=False))
    bh = O.dequantize(qw["codes"], qw["scales"], block=(16, 16))
    ah = O.dequantize(qx["codes"][rows], qx["scales"][rows])
    ref = O.gemm(ah, bh, s_dec_a=qx["s_dec"], s_dec_b=qw["s_dec"])
    got = out[torch.from_numpy(rows).cuda()].cpu().numpy()
    assert rel_fro(got, ref) <= TOL


@pytest.mark.parametrize("mnk", [(4096, 4096, 16384), (1024, 768, 16384)])
def test_gemm_long_k_sampled_rows(gpu_lib, mnk):
    """A weight-gradient-like product (long contraction, FP32 output, 3.46
    and 0.21 waves of tiles on the persistent grid): sampled rows against the
    float64 oracle over the full contraction, and the same bits on a second
    call."""
    F = gpu_lib
    M, N, K = mnk
    a = S.normal((M, K), 1e-3, seed=21)
    b = S.sparse_outliers(N, K, seed=22)
    qa, qb = O.nvfp4_quantize_1d(S.as_f32(a)), O.nvfp4_quantize_1d(S.as_f32(b))
    ta, tb = upload_qtensor(F, qa, M, K, 0, 0), upload_qtensor(F, qb, N, K, 0, 0)
    out = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ws = F.Workspace(M, N, K)
    F.fp4_gemm(ta, tb, out, ws=ws)
    again = torch.full_like(out, float("nan"))
    F.fp4_gemm(ta, tb, again, ws=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    assert torch.equal(out, again)
    rows = np.sort(np.random.default_rng(6).choice(M, 32, replace=False))
    bh = O.dequantize(qb["codes"], qb["scales"])
    ah = O.dequantize(qa["codes"][rows], qa["scales"][rows])
    ref = O.gemm(ah, bh, s_dec_a=qa["s_dec"], s_dec_b=qb["s_dec"])
    got = out[torch.from_numpy(rows).cuda()].cpu().numpy()
    assert rel_fro(got, ref) <= TOL


@pytest.mark.parametrize("mnk", SHAPES)
def test_gemm_mxfp4_small_shapes(gpu_lib, mnk):
    _small(gpu_lib, 1, mnk)
