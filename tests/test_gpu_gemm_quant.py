"""fp4_gemm_quant / fp4_gemm_quant_ex: the GEMM with its FP32 result encoded
to NVFP4 1x16 (RTN or SR, supplied tensor amax) in the epilogue, optionally
also stored as BF16.

Exact parity: MXFP4 operands whose values lie on the E2M1 grid with block
scale 2^0 (every 32-block holds a 4, so floor(log2 4) - 2 = 0) make every
partial sum a multiple of 1/4 far below 2^24, so the FP32 accumulation is
exact in any order and the result equals the float64 product; the encode
must then match the oracle's NVFP4 quantization of that product bit for bit.
General NVFP4 data is checked against the float64 GEMM within the NVFP4
quantization error."""
import numpy as np
import pytest
import torch

import fqt_synth as S
import oracle as O
from fp4_testlib import from_mma_layout, rel_fro

pytestmark = pytest.mark.gpu

LEVELS = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)


def _grid_operand(rows, cols, seed):
    rng = np.random.default_rng(seed)
    x = LEVELS[rng.integers(0, 8, (rows, cols))] * rng.choice([-1.0, 1.0], (rows, cols))
    x = x.astype(np.float32)
    x[:, ::32] = 4.0                      # block max 4 in every 32-block
    return x


def _mx(F, x):
    R, Cc = x.shape
    q = F.QTensor.empty(R, Cc, F.MXFP4)
    F.fp4_quantize(torch.from_numpy(x).to(torch.bfloat16).cuda(), q, fmt=F.MXFP4, ws=F.Workspace())
    return q


@pytest.mark.parametrize("mnk", [(256, 384, 512), (128, 256, 64), (384, 128, 256)])
@pytest.mark.parametrize("amax_scale", [1.0, 0.5, 3.0])
def test_gemm_quant_exact_against_oracle(gpu_lib, mnk, amax_scale):
    F = gpu_lib
    M, N, K = mnk
    a, b = _grid_operand(M, K, 1), _grid_operand(N, K, 2)
    qa, qb = _mx(F, a), _mx(F, b)
    c64 = a.astype(np.float64) @ b.astype(np.float64).T
    c32 = c64.astype(np.float32)
    assert np.array_equal(c32.astype(np.float64), c64)        # the product is exact in FP32
    amax = np.float32(np.abs(c32).max() * amax_scale)
    out = F.QTensor.empty(M, N, F.NVFP4)
    amax_in = torch.tensor([amax], dtype=torch.float32, device="cuda")
    c_amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    ws = F.Workspace(M, N, K)
    F.fp4_gemm_quant(qa, qb, out, amax_in, c_amax=c_amax, ws=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    ref = O.nvfp4_quantize_1d(c32, amax_in=float(amax))
    assert np.array_equal(out.codes.cpu().numpy().reshape(M, N // 2), ref["codes"])
    assert np.array_equal(out.scales.cpu().numpy().reshape(M, N // 16), ref["scales"])
    assert np.array_equal(from_mma_layout(out.scales_mma.cpu().numpy(), M, N // 16), ref["scales"])
    assert float(out.s_dec.item()) == float(ref["s_dec"])
    assert float(out.amax.item()) == float(amax)
    assert float(c_amax.item()) == float(np.abs(c32).max())


@pytest.mark.parametrize("mnk", [(256, 384, 512), (384, 128, 256)])
@pytest.mark.parametrize("with_bf16", [False, True])
def test_gemm_quant_sr_exact_against_oracle(gpu_lib, mnk, with_bf16):
    """fp4_gemm_quant_ex with stochastic rounding: on exact products the
    codes, both scale layouts, s_dec and amax match the oracle's NVFP4 SR
    quantization of the product (16-bit draws of the output's element index,
    seed 5, stream 9) bit for bit; the optional BF16 copy equals the product
    rounded to BF16 (exactly what fp4_gemm writes)."""
    F = gpu_lib
    M, N, K = mnk
    a, b = _grid_operand(M, K, 3), _grid_operand(N, K, 4)
    qa, qb = _mx(F, a), _mx(F, b)
    c32 = (a.astype(np.float64) @ b.astype(np.float64).T).astype(np.float32)
    amax = np.float32(np.abs(c32).max())
    out = F.QTensor.empty(M, N, F.NVFP4)
    amax_in = torch.tensor([amax], dtype=torch.float32, device="cuda")
    c_amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    y = torch.full((M, N + 64), 7.0, dtype=torch.bfloat16, device="cuda") if with_bf16 else None
    ws = F.Workspace(M, N, K)
    F.fp4_gemm_quant_ex(qa, qb, out, amax_in, round=F.SR, sr_seed=5, sr_stream=9,
                        c_bf16=y[:, :N] if with_bf16 else None, c_amax=c_amax, ws=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    ref = O.nvfp4_quantize_1d(c32, "sr", sr_seed=5, sr_stream=9, amax_in=float(amax))
    assert np.array_equal(out.codes.cpu().numpy().reshape(M, N // 2), ref["codes"])
    assert np.array_equal(out.scales.cpu().numpy().reshape(M, N // 16), ref["scales"])
    assert np.array_equal(from_mma_layout(out.scales_mma.cpu().numpy(), M, N // 16), ref["scales"])
    assert float(out.s_dec.item()) == float(ref["s_dec"])
    assert float(c_amax.item()) == float(amax)
    if with_bf16:
        want = torch.from_numpy(c32).to(torch.bfloat16)
        assert torch.equal(y[:, :N].cpu(), want)
        assert (y[:, N:] == 7.0).all()                       # nothing beyond N is touched
        # the row-wise RTN mode with the copy keeps its own encode unchanged
        out_rtn = F.QTensor.empty(M, N, F.NVFP4)
        F.fp4_gemm_quant_ex(qa, qb, out_rtn, amax_in, c_bf16=y[:, :N], ws=ws)
        torch.cuda.synchronize()
        ref_rtn = O.nvfp4_quantize_1d(c32, amax_in=float(amax))
        assert np.array_equal(out_rtn.codes.cpu().numpy().reshape(M, N // 2), ref_rtn["codes"])


def test_gemm_quant_nvfp4_llama_like_within_quantization_error(gpu_lib):
    F = gpu_lib
    M, N, K = 512, 768, 1024
    x = S.as_f32(S.student_t_channels(M, K, seed=3)[0])
    w = S.as_f32(S.normal((N, K), 0.02, seed=4))
    qx_ref, qw_ref = O.nvfp4_quantize_1d(x), O.nvfp4_quantize_2d(w)
    c64 = O.gemm(O.dequantize(qx_ref["codes"], qx_ref["scales"]),
                 O.dequantize(qw_ref["codes"], qw_ref["scales"], (16, 16)),
                 s_dec_a=qx_ref["s_dec"], s_dec_b=qw_ref["s_dec"])
    qa = F.QTensor.empty(M, K)
    qb = F.QTensor.empty(N, K, F.NVFP4, F.BLOCK_2D)
    ws = F.Workspace(M, N, K)
    F.fp4_quantize(torch.from_numpy(x).to(torch.bfloat16).cuda(), qa, ws=ws)
    F.fp4_quantize(torch.from_numpy(w).to(torch.bfloat16).cuda(), qb, block=F.BLOCK_2D, ws=ws)
    amax = float(np.abs(c64).max())
    out = F.QTensor.empty(M, N, F.NVFP4)
    F.fp4_gemm_quant(qa, qb, out, torch.tensor([amax], dtype=torch.float32, device="cuda"), ws=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    deq = O.dequantize(out.codes.cpu().numpy().reshape(M, N // 2),
                       out.scales.cpu().numpy().reshape(M, N // 16)) * float(out.s_dec.item())
    err = rel_fro(deq, c64)
    assert err < 0.15                     # NVFP4 RTN noise of the output (about 0.1)
    ref = O.nvfp4_quantize_1d(c64.astype(np.float32), amax_in=amax)
    codes = out.codes.cpu().numpy().reshape(M, N // 2)
    assert np.mean(codes != ref["codes"]) < 0.01  # only FP32-vs-float64 rounding flips


def test_gemm_quant_rejects_bad_arguments(gpu_lib):
    F = gpu_lib
    a = F.QTensor.empty(128, 128)
    b = F.QTensor.empty(128, 128)
    wrong = F.QTensor.empty(128, 256)
    amax = torch.ones(1, device="cuda")
    with pytest.raises(F.Fp4Error):
        F.fp4_gemm_quant(a, b, wrong, amax)
    good = F.QTensor.empty(128, 128)
    with pytest.raises(F.Fp4Error) as e:                       # unknown rounding
        F.fp4_gemm_quant_ex(a, b, good, amax, round=2)
    assert e.value.code == 4
    narrow = torch.empty((128, 120), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(F.Fp4Error) as e:                       # BF16 copy narrower than N
        F.fp4_gemm_quant_ex(a, b, good, amax, c_bf16=narrow)
    assert e.value.code == 3
    mx = F.QTensor.empty(128, 128, F.MXFP4)
    with pytest.raises(F.Fp4Error):
        F.fp4_gemm_quant(a, b, mx, amax)
