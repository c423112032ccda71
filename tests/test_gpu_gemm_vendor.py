"""fp4_gemm against an independent implementation: the vendor's block-scaled
NVFP4 GEMM (cuBLASLt through torch.nn.functional.scaled_mm), given the very
operand bytes fp4_gemm reads (E2M1 codes, E4M3 block scales in the 128-row x
4-block atom layout, FP32 tensor scales), and the same for MXFP4 (E8M0 1x32
block scales, tensor scale 1) against the vendor's MX recipe.  Both
accumulate in FP32 and round once to BF16; with the kernels the vendor picks
on B200 the two products are identical element for element (reported), and
the test requires agreement within one BF16 rounding of the product, since
which vendor kernel runs (and its accumulation order) is the vendor's choice.
The vendor kernel is used here and in `bench.py --case gemm_vendor` only, as
a cross-check and a rate to compare with, never on the library's path."""
import pytest
import torch

import fqt_synth as S

pytestmark = pytest.mark.gpu

Fn = torch.nn.functional


def _agree(y, yv):
    """Equal, or apart by at most one BF16 unit (2^-7 of each element) plus an
    absolute floor of 2^-12 of the largest output for elements that cancel:
    what a different FP32 accumulation order can change.  A wrong product
    (operand, scale or layout) is off by far more."""
    if torch.equal(y, yv):
        print("bit-identical")
        return
    a, b = y.float(), yv.float()
    tol = torch.maximum(a.abs(), b.abs()) * 2.0 ** -7 + a.abs().max() * 2.0 ** -12
    assert bool(((a - b).abs() <= tol).all())


def _vendor(qa, qb):
    M, N, K = qa.rows, qb.rows, qa.cols
    fp4 = torch.float4_e2m1fn_x2
    ST, SW = Fn.ScalingType, Fn.SwizzleType
    return Fn.scaled_mm(qa.codes.view(M, K // 2).view(fp4), qb.codes.view(N, K // 2).view(fp4).t(),
                        [qa.scales_mma.view(torch.float8_e4m3fn), qa.s_dec],
                        [ST.BlockWise1x16, ST.TensorWise],
                        [qb.scales_mma.view(torch.float8_e4m3fn), qb.s_dec],
                        [ST.BlockWise1x16, ST.TensorWise],
                        swizzle_a=[SW.SWIZZLE_32_4_4, SW.NO_SWIZZLE],
                        swizzle_b=[SW.SWIZZLE_32_4_4, SW.NO_SWIZZLE],
                        output_dtype=torch.bfloat16)


@pytest.mark.parametrize("M,N,K,w_block", [(256, 512, 1024, "1d"), (384, 640, 512, "2d"),
                                           (1024, 768, 4096, "2d"), (128, 384, 320, "1d"),
                                           (8192, 4096, 8192, "2d")])
def test_fp4_gemm_equals_vendor_nvfp4_gemm(gpu_lib, M, N, K, w_block):
    if not hasattr(Fn, "scaled_mm") or not hasattr(torch, "float4_e2m1fn_x2"):
        pytest.skip("this torch has no NVFP4 scaled_mm")
    F = gpu_lib
    dev = torch.device("cuda", 0)
    blk = F.BLOCK_2D if w_block == "2d" else F.BLOCK_1D
    x = S.student_t_channels(M, K, seed=M + K)[0].to(dev)
    w = S.normal((N, K), 0.02, seed=N + K).to(dev)
    qa = F.QTensor.empty(M, K, device=dev, logical_scales=False)
    qb = F.QTensor.empty(N, K, F.NVFP4, blk, device=dev, logical_scales=False)
    ws = F.Workspace(M, N, K, device=dev)
    F.fp4_quantize(x, qa, ws=ws)
    F.fp4_quantize(w, qb, block=blk, ws=ws)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev)
    F.fp4_gemm(qa, qb, y, ws=ws)
    yv = _vendor(qa, qb)
    torch.cuda.synchronize()
    assert ws.status() == 0
    assert torch.isfinite(y).all()
    _agree(y, yv)


def _vendor_mx(qa, qb):
    M, N, K = qa.rows, qb.rows, qa.cols
    fp4 = torch.float4_e2m1fn_x2
    ST, SW = Fn.ScalingType, Fn.SwizzleType
    return Fn.scaled_mm(qa.codes.view(M, K // 2).view(fp4), qb.codes.view(N, K // 2).view(fp4).t(),
                        qa.scales_mma.view(torch.float8_e8m0fnu), ST.BlockWise1x32,
                        qb.scales_mma.view(torch.float8_e8m0fnu), ST.BlockWise1x32,
                        swizzle_a=SW.SWIZZLE_32_4_4, swizzle_b=SW.SWIZZLE_32_4_4,
                        output_dtype=torch.bfloat16)


@pytest.mark.parametrize("M,N,K,quest", [(256, 512, 1024, False), (384, 640, 512, False),
                                         (1024, 768, 4096, True), (128, 384, 256, False)])
def test_fp4_gemm_equals_vendor_mxfp4_gemm(gpu_lib, M, N, K, quest):
    if not hasattr(Fn, "scaled_mm") or not hasattr(torch, "float8_e8m0fnu"):
        pytest.skip("this torch has no MXFP4 scaled_mm")
    F = gpu_lib
    dev = torch.device("cuda", 0)
    x = S.student_t_channels(M, K, seed=M + K + 7)[0].to(dev)
    w = S.normal((N, K), 0.02, seed=N + K + 7).to(dev)
    qa = F.QTensor.empty(M, K, F.MXFP4, device=dev, logical_scales=False)
    qb = F.QTensor.empty(N, K, F.MXFP4, device=dev, logical_scales=False)
    ws = F.Workspace(M, N, K, device=dev)
    F.fp4_quantize(x, qa, fmt=F.MXFP4, round=F.QUEST if quest else F.RTN, rht_n=32 if quest else 0,
                   rht_seed=5, ws=ws)
    F.fp4_quantize(w, qb, fmt=F.MXFP4, rht_n=32 if quest else 0, rht_seed=5, ws=ws)
    assert float(qa.s_dec.item()) == 1.0 and float(qb.s_dec.item()) == 1.0
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev)
    F.fp4_gemm(qa, qb, y, ws=ws)
    yv = _vendor_mx(qa, qb)
    torch.cuda.synchronize()
    assert ws.status() == 0
    assert torch.isfinite(y).all()
    _agree(y, yv)
