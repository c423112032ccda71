"""The C-ABI library loads on a machine without a GPU, exports every symbol
include/fp4.h declares, and rejects bad arguments before touching CUDA."""
import ctypes as C
import os
import re

import pytest

import fp4_fully_quantized_b200 as F
from conftest import ROOT


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "fp4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", src)
    keep = [n for n in names if n.startswith(("fp4_", "fqt_"))]
    return sorted(set(keep))


@pytest.fixture(scope="module")
def lib():
    from fp4_fully_quantized_b200 import build
    build.build()
    return F.load()


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert set(declared) == set(F.EXPORTS), (declared, F.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_host_only_helpers(lib):
    assert lib.fp4_abi_version() == 1
    assert lib.fp4_status_str(7) == b"a tensor amax was Inf or NaN"
    assert F.qtensor_sizes(256, 512, F.NVFP4, F.BLOCK_1D) == (256 * 256, 256 * 32, 256 * 32)
    assert F.qtensor_sizes(256, 512, F.NVFP4, F.BLOCK_2D)[1] == 16 * 32
    assert F.qtensor_sizes(128, 96, F.MXFP4, F.BLOCK_1D) == (128 * 48, 128 * 3, 128 * 4)
    assert F.qtensor_sizes(100, 64, F.NVFP4, F.BLOCK_1D)[2] == 128 * 4
    assert lib.fp4_workspace_bytes(128, 128, 64) >= 256
    nv = F.linear_cfg(F.NVFP4)
    assert (nv.w_block, nv.round_fwd, nv.round_bwd, nv.round_x_t, nv.rht_mask) == (
        F.BLOCK_2D, F.RTN, F.SR, F.SR, 0)
    mx = F.linear_cfg(F.MXFP4)
    assert (mx.w_block, mx.round_bwd, mx.rht_mask, mx.rht_n) == (F.BLOCK_1D, F.RTN, 7, 32)


def _q(rows, cols, fmt=0, block=0):
    return F.QTensorC(C.c_void_p(4096), C.c_void_p(4096), C.c_void_p(4096), C.c_void_p(4096),
                      C.c_void_p(4100), rows, cols, fmt, block)


def test_argument_errors_return_before_launch(lib):
    p = F.QParamsC()
    lib.fp4_qparams_default(C.byref(p))
    q = _q(32, 64)
    fake_x = C.c_void_p(1 << 20)
    # no output at all
    assert lib.fp4_quantize(fake_x, 32, 64, 64, C.byref(p), None, None, None, 0, None) == 1
    # misaligned input / leading dimension
    assert lib.fp4_quantize(C.c_void_p((1 << 20) + 2), 32, 64, 64, C.byref(p), C.byref(q), None,
                            None, 0, None) == 3
    assert lib.fp4_quantize(fake_x, 32, 64, 66, C.byref(p), C.byref(q), None, None, 0, None) == 3
    # cols not a multiple of 16
    q2 = _q(32, 40)
    assert lib.fp4_quantize(fake_x, 32, 40, 40, C.byref(p), C.byref(q2), None, None, 0, None) == 2
    # qtensor shape disagrees with the request
    assert lib.fp4_quantize(fake_x, 32, 128, 128, C.byref(p), C.byref(q), None, None, 0, None) == 2
    # 2-D blocks are NVFP4 only; bad Hadamard size; bad rounding
    p2 = F.QParamsC(); lib.fp4_qparams_default(C.byref(p2)); p2.fmt = 1; p2.block = 1
    assert lib.fp4_quantize(fake_x, 32, 64, 64, C.byref(p2), C.byref(q), None, None, 0, None) == 4
    p3 = F.QParamsC(); lib.fp4_qparams_default(C.byref(p3)); p3.rht_n = 8
    assert lib.fp4_quantize(fake_x, 32, 64, 64, C.byref(p3), C.byref(q), None, None, 0, None) == 4
    p4 = F.QParamsC(); lib.fp4_qparams_default(C.byref(p4)); p4.round = 5
    assert lib.fp4_quantize(fake_x, 32, 64, 64, C.byref(p4), C.byref(q), None, None, 0, None) == 4
    # workspace too small
    assert lib.fp4_quantize(fake_x, 32, 64, 64, C.byref(p), C.byref(q), None, C.c_void_p(4096), 8,
                            None) == 5
    # GEMM: shape rules (M, N multiples of 128; K multiple of 64), formats, workspace
    a, b = _q(128, 128), _q(256, 128)
    ws = C.c_void_p(1 << 21)
    c = C.c_void_p(1 << 22)
    assert lib.fp4_gemm(C.byref(_q(96, 128)), C.byref(b), 1.0, c, 256, 1, None, ws, 256, None) == 2
    assert lib.fp4_gemm(C.byref(a), C.byref(_q(256, 96)), 1.0, c, 256, 1, None, ws, 256, None) == 2
    assert lib.fp4_gemm(C.byref(a), C.byref(_q(256, 128, 1)), 1.0, c, 256, 1, None, ws, 256,
                        None) == 4
    assert lib.fp4_gemm(C.byref(a), C.byref(b), 1.0, c, 200, 1, None, ws, 256, None) == 3
    assert lib.fp4_gemm(C.byref(a), C.byref(b), 1.0, c, 256, 1, None, None, 0, None) == 5
    assert lib.fp4_gemm(C.byref(a), C.byref(b), 1.0, c, 256, 7, None, ws, 256, None) == 4
    # linear layer: 2-D weights cannot take a rotation on fprop/dgrad
    cfg = F.linear_cfg(F.NVFP4, rht_mask=F.RHT_FPROP)
    assert lib.fqt_linear_fwd(C.byref(cfg), 128, 128, 128, fake_x, fake_x, fake_x,
                              C.byref(F.SavedC()), ws, 256, None) == 9


def test_gemm_quant_and_noise_argument_errors(lib):
    """The epilogue-quantized GEMM and the noise diagnostic validate on the
    host and return before any launch."""
    a, b = _q(128, 128), _q(256, 128)
    out = _q(128, 256)
    amax = C.c_void_p(1 << 23)
    ws = C.c_void_p(1 << 21)
    # missing supplied amax / output
    assert lib.fp4_gemm_quant(C.byref(a), C.byref(b), 1.0, None, C.byref(out), None, ws, 256,
                              None) == 1
    assert lib.fp4_gemm_quant(C.byref(a), C.byref(b), 1.0, amax, None, None, ws, 256, None) == 1
    # output must be NVFP4 1x16 of shape [M, N]
    assert lib.fp4_gemm_quant(C.byref(a), C.byref(b), 1.0, amax, C.byref(_q(128, 256, 1)), None,
                              ws, 256, None) == 4
    assert lib.fp4_gemm_quant(C.byref(a), C.byref(b), 1.0, amax, C.byref(_q(128, 256, 0, 1)), None,
                              ws, 256, None) == 4
    assert lib.fp4_gemm_quant(C.byref(a), C.byref(b), 1.0, amax, C.byref(_q(256, 256)), None,
                              ws, 256, None) == 2
    # GEMM shape rules still apply
    assert lib.fp4_gemm_quant(C.byref(_q(96, 128)), C.byref(b), 1.0, amax, C.byref(_q(96, 256)),
                              None, ws, 256, None) == 2
    # workspace
    assert lib.fp4_gemm_quant(C.byref(a), C.byref(b), 1.0, amax, C.byref(out), None, None, 0,
                              None) == 5
    # noise diagnostic: null sums, shape mismatch, misaligned sums, bad format
    x = C.c_void_p(1 << 20)
    q = _q(32, 64)
    sums = C.c_void_p(1 << 24)
    assert lib.fp4_quant_noise(x, 32, 64, 64, C.byref(q), None, None, 0, None) == 1
    assert lib.fp4_quant_noise(x, 32, 128, 128, C.byref(q), sums, None, 0, None) == 2
    assert lib.fp4_quant_noise(x, 32, 64, 64, C.byref(q), C.c_void_p((1 << 24) + 4), None, 0,
                               None) == 3
    assert lib.fp4_quant_noise(x, 32, 64, 64, C.byref(_q(32, 64, 5)), sums, None, 0, None) == 4


def test_linear_layer_rejects_before_any_launch(lib):
    """fqt_linear_fwd / fqt_linear_bwd check every one of their quantize and
    GEMM calls before enqueuing the first: a shape only the GEMM rejects
    (M = 96, not a multiple of 128) returns FP4_ERR_SHAPE, not the CUDA error
    the X quantizer's first enqueue would meet on a machine without a GPU, and
    the library's launch counter does not move."""
    M, N, K = 96, 128, 128
    sv = F.SavedC(_q(M, K), _q(K, M), _q(N, K, 0, 1), _q(K, N, 0, 1), _q(M, N), _q(N, M))
    cfg = F.linear_cfg(F.NVFP4)
    x = C.c_void_p(1 << 20)
    ws = C.c_void_p(1 << 21)
    n0 = lib.fp4_kernel_launches()
    assert lib.fqt_linear_fwd(C.byref(cfg), M, N, K, x, x, x, C.byref(sv), ws, 256, None) == 2
    assert lib.fqt_linear_bwd(C.byref(cfg), M, N, K, x, C.byref(sv), x, x, ws, 256, None) == 2
    # a missing workspace is only a GEMM error too
    sv2 = F.SavedC(_q(128, K), _q(K, 128), _q(N, K, 0, 1), _q(K, N, 0, 1), _q(128, N), _q(N, 128))
    assert lib.fqt_linear_fwd(C.byref(cfg), 128, N, K, x, x, x, C.byref(sv2), None, 0, None) == 5
    assert lib.fp4_kernel_launches() == n0


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without the built library every entry point raises: there is no CPU
    fallback behind the binding."""
    import torch
    monkeypatch.setattr(F, "LIB_PATH", str(tmp_path / "libfp4fqt.so"))
    monkeypatch.setattr(F, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        F.load()
    with pytest.raises(RuntimeError, match="missing"):
        F.qtensor_sizes(16, 16)
    with pytest.raises(RuntimeError, match="missing"):
        F.linear_cfg(F.NVFP4)
    x = torch.zeros((16, 16), dtype=torch.bfloat16)
    with pytest.raises((RuntimeError, AssertionError)):
        F.fp4_quantize(x, None)


def test_gemm_rejects_tile_counts_beyond_32_bits(lib):
    """Shapes within the per-dimension limits whose 128 x 256 tile count does
    not fit the kernel's 32-bit tile numbering are rejected on the host."""
    big = 1 << 30
    a, b = _q(big, 128), _q(big, 128)
    c = C.c_void_p(1 << 22)
    ws = C.c_void_p(1 << 21)
    assert lib.fp4_gemm(C.byref(a), C.byref(b), 1.0, c, big, 0, None, ws, 256, None) == 2
    out = _q(big, big)
    amax = C.c_void_p(1 << 23)
    assert lib.fp4_gemm_quant(C.byref(a), C.byref(b), 1.0, amax, C.byref(out), None, ws, 256,
                              None) == 2
    # just above the limit of 2^30 tiles: 2^23 row blocks x (2^7 + 1) column blocks
    b2 = _q((1 << 15) + 256, 128)
    assert lib.fp4_gemm(C.byref(a), C.byref(b2), 1.0, c, (1 << 15) + 256, 0, None, ws, 256,
                        None) == 2


def test_allreduce_argument_checks(lib):
    """fp4_allreduce_sum_f32 validates before touching NCCL: no communicator,
    a negative count, a misaligned buffer; an empty sum does nothing."""
    comm = C.c_void_p(1 << 20)
    assert lib.fp4_allreduce_sum_f32(None, C.c_void_p(1 << 21), 4, None) == 1
    assert lib.fp4_allreduce_sum_f32(comm, C.c_void_p(1 << 21), -1, None) == 2
    assert lib.fp4_allreduce_sum_f32(comm, C.c_void_p((1 << 21) + 2), 4, None) == 3
    assert lib.fp4_allreduce_sum_f32(comm, None, 0, None) == 0
