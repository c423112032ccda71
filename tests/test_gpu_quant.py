"""GPU quantizers vs the CPU oracle, element by element (bit-exact codes,
scales, amax and s_dec), through the C ABI.

Covers NVFP4 1x16 (RTN and Philox SR, with and without the 16-point random
Hadamard transform), the transposed (column) quantizer used for wgrad,
NVFP4 16x16 2-D weight tiles, MXFP4 1x32 (with the 32-point transform),
supplied amax, edge cases (empty, all-zero, subnormal and huge values,
ragged sizes) and sampled rows of the Llama-7B-shaped activations.
"""
import numpy as np
import pytest
import torch

import fqt_synth as S
import oracle as O
from fp4_testlib import expand_2d, from_mma_layout, unpack_codes

pytestmark = pytest.mark.gpu


def _gpu_quant(F, x, fmt, block=0, round=0, round_t=0, rht_n=0, rht_n_t=0, seed=0, stream=0,
               stream_t=0, row=True, col=False, amax_in=None):
    R, Cc = x.shape
    xd = x.cuda()
    out = F.QTensor.empty(R, Cc, fmt, block) if row else None
    out_t = F.QTensor.empty(Cc, R, fmt, block) if col else None
    ws = F.Workspace()
    ain = None if amax_in is None else torch.tensor([amax_in], dtype=torch.float32, device="cuda")
    F.fp4_quantize(xd, out, out_t, fmt=fmt, block=block, round=round, round_t=round_t,
                   rht_n=rht_n, rht_n_t=rht_n_t, rht_seed=seed, sr_seed=seed, sr_stream=stream,
                   sr_stream_t=stream_t, amax_in=ain, ws=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    return out, out_t


def _np(t):
    return t.cpu().numpy()


def _check_1d(q, ref, fmt):
    R, Cc = q.rows, q.cols
    bs = 32 if fmt == 1 else 16
    codes = _np(q.codes).reshape(R, Cc // 2)
    bad = np.argwhere(codes != ref["codes"])
    assert bad.size == 0, f"{len(bad)} code bytes differ, first {bad[:4].tolist()}"
    sc = _np(q.scales).reshape(R, Cc // bs)
    assert np.array_equal(sc, ref["scales"])
    assert np.array_equal(from_mma_layout(_np(q.scales_mma), R, Cc // bs), ref["scales"])
    assert float(_np(q.s_dec)[0]) == float(ref["s_dec"])
    if fmt == 0:
        assert float(_np(q.amax)[0]) == float(ref["amax"])


RTN, SR = 0, 1


@pytest.mark.parametrize("shape", [(128, 256), (48, 80), (256, 4096), (16, 16), (1, 32)])
@pytest.mark.parametrize("rnd", [RTN, SR])
@pytest.mark.parametrize("rht", [0, 16])
def test_nvfp4_rows(gpu_lib, shape, rnd, rht):
    F = gpu_lib
    R, Cc = shape
    if rht and Cc % rht:
        pytest.skip("Hadamard block must divide the row")
    x = S.sparse_outliers(R, Cc, seed=R + Cc)
    q, _ = _gpu_quant(F, x, 0, round=rnd, rht_n=rht, seed=5, stream=7)
    ref = O.nvfp4_quantize_1d(S.as_f32(x), "sr" if rnd else "rtn", rht_n=rht, rht_seed=5,
                              sr_seed=5, sr_stream=7)
    _check_1d(q, ref, 0)


@pytest.mark.parametrize("shape", [(128, 256), (64, 64), (96, 48), (256, 1024), (32, 80)])
@pytest.mark.parametrize("rnd", [RTN, SR])
@pytest.mark.parametrize("rht", [0, 16])
def test_nvfp4_transposed(gpu_lib, shape, rnd, rht):
    F = gpu_lib
    R, Cc = shape
    if rht and R % rht:
        pytest.skip("Hadamard block must divide the blocked dimension")
    x, _ = S.outlier_columns(R, Cc, seed=3)
    _, qt = _gpu_quant(F, x, 0, round_t=rnd, rht_n_t=rht, seed=11, stream_t=3, row=False, col=True)
    xt = np.ascontiguousarray(S.as_f32(x).T)
    ref = O.nvfp4_quantize_1d(xt, "sr" if rnd else "rtn", rht_n=rht, rht_seed=11, sr_seed=11,
                              sr_stream=3)
    _check_1d(qt, ref, 0)


@pytest.mark.parametrize("shape", [(128, 256), (48, 80), (1024, 4096), (16, 16), (64, 272)])
def test_nvfp4_row_and_transposed_together(gpu_lib, shape):
    """Row-wise RTN + transposed SR with a 16-point Hadamard on the transposed
    operand (the wgrad-RHT layer's X and dY): both amaxes come from one read."""
    F = gpu_lib
    x, _ = S.outlier_columns(*shape, seed=0)
    q, qt = _gpu_quant(F, x, 0, round=RTN, round_t=SR, rht_n_t=16, seed=0, stream_t=3, col=True)
    xf = S.as_f32(x)
    _check_1d(q, O.nvfp4_quantize_1d(xf), 0)
    _check_1d(qt, O.nvfp4_quantize_1d(np.ascontiguousarray(xf.T), "sr", rht_n=16, rht_seed=0,
                                      sr_seed=0, sr_stream=3), 0)


@pytest.mark.parametrize("shape", [(128, 256), (48, 80), (1024, 512), (64, 272)])
@pytest.mark.parametrize("rht_t", [0, 16])
@pytest.mark.parametrize("rnd,rnd_t", [(RTN, RTN), (RTN, SR), (SR, RTN), (SR, SR)])
def test_nvfp4_dual_with_rotated_rows(gpu_lib, shape, rht_t, rnd, rnd_t):
    """The fused row-wise + transposed NVFP4 quantizer with the 16-point
    Hadamard transform on the row-wise output (and with or without it on the
    transposed one), every pair of roundings: both outputs bit-exact."""
    F = gpu_lib
    x, _ = S.outlier_columns(*shape, seed=5)
    q, qt = _gpu_quant(F, x, 0, round=rnd, round_t=rnd_t, rht_n=16, rht_n_t=rht_t, seed=9,
                       stream=1, stream_t=2, col=True)
    xf = S.as_f32(x)
    m = lambda r: "sr" if r == SR else "rtn"
    _check_1d(q, O.nvfp4_quantize_1d(xf, m(rnd), rht_n=16, rht_seed=9, sr_seed=9, sr_stream=1), 0)
    _check_1d(qt, O.nvfp4_quantize_1d(np.ascontiguousarray(xf.T), m(rnd_t), rht_n=rht_t,
                                      rht_seed=9, sr_seed=9, sr_stream=2), 0)


@pytest.mark.parametrize("shape", [(256, 256), (48, 96), (4096, 512)])
def test_nvfp4_2d(gpu_lib, shape):
    F = gpu_lib
    R, Cc = shape
    w = S.normal(shape, 0.02, seed=R)
    q, qt = _gpu_quant(F, w, 0, block=1, col=True)
    ref = O.nvfp4_quantize_2d(S.as_f32(w))
    reft = O.nvfp4_quantize_2d(np.ascontiguousarray(S.as_f32(w).T))
    for t, r, rows, cols in ((q, ref, R, Cc), (qt, reft, Cc, R)):
        assert np.array_equal(_np(t.codes).reshape(rows, cols // 2), r["codes"])
        assert np.array_equal(_np(t.scales).reshape(rows // 16, cols // 16), r["scales"])
        assert np.array_equal(from_mma_layout(_np(t.scales_mma), rows, cols // 16),
                              expand_2d(r["scales"], rows))
        assert float(_np(t.s_dec)[0]) == float(r["s_dec"])
        assert float(_np(t.amax)[0]) == float(r["amax"])


@pytest.mark.parametrize("shape", [(128, 256), (64, 96), (256, 4096)])
@pytest.mark.parametrize("rnd", [RTN, SR])
@pytest.mark.parametrize("rht", [0, 32])
def test_mxfp4_rows_and_transposed(gpu_lib, shape, rnd, rht):
    F = gpu_lib
    R, Cc = shape
    if rht and (Cc % rht or R % rht):
        pytest.skip("Hadamard block must divide the blocked dimension")
    x = S.sparse_outliers(R, Cc, seed=9)
    q, qt = _gpu_quant(F, x, 1, round=rnd, round_t=rnd, rht_n=rht, rht_n_t=rht, seed=2, stream=4,
                       stream_t=5, col=True)
    xf = S.as_f32(x)
    kw = dict(round_mode="sr" if rnd else "rtn", rht_n=rht, rht_seed=2, sr_seed=2)
    _check_1d(q, O.mxfp4_quantize(xf, sr_stream=4, **kw), 1)
    _check_1d(qt, O.mxfp4_quantize(np.ascontiguousarray(xf.T), sr_stream=5, **kw), 1)


@pytest.mark.parametrize("shape", [(128, 256), (64, 96), (256, 4096), (32, 64)])
@pytest.mark.parametrize("rht", [0, 32])
@pytest.mark.parametrize("with_t", [False, True])
def test_mxfp4_quest_rows(gpu_lib, shape, rht, with_t):
    """MXFP4 with the QuEST-style forward scale on the row-wise output, alone
    (row kernel) and beside a round-to-nearest transposed output (fused
    kernel): codes and scales bit-exact with the oracle."""
    F = gpu_lib
    R, Cc = shape
    if rht and (Cc % rht or (with_t and R % rht)):
        pytest.skip("Hadamard block must divide the blocked dimension")
    x = S.sparse_outliers(R, Cc, seed=13)
    q, qt = _gpu_quant(F, x, 1, round=F.QUEST, round_t=RTN, rht_n=rht, rht_n_t=rht, seed=4,
                       col=with_t)
    xf = S.as_f32(x)
    _check_1d(q, O.mxfp4_quantize(xf, "quest", rht_n=rht, rht_seed=4), 1)
    if with_t:
        _check_1d(qt, O.mxfp4_quantize(np.ascontiguousarray(xf.T), rht_n=rht, rht_seed=4), 1)


def test_quest_requests_outside_mxfp4_rows_are_rejected(gpu_lib):
    F = gpu_lib
    x = S.normal((64, 64), 1.0, seed=1).cuda()
    with pytest.raises(F.Fp4Error) as e:
        F.fp4_quantize(x, F.QTensor.empty(64, 64), round=F.QUEST)            # NVFP4
    assert e.value.code == 9
    with pytest.raises(F.Fp4Error) as e:
        F.fp4_quantize(x, None, F.QTensor.empty(64, 64, F.MXFP4), fmt=F.MXFP4, round_t=F.QUEST)
    assert e.value.code == 9


@pytest.mark.parametrize("case", ["nvfp4_rtn", "nvfp4_sr", "nvfp4_2d", "mxfp4", "nvfp4_ragged"])
def test_quant_noise_matches_oracle(gpu_lib, case):
    """fp4_quant_noise (sum x^2, sum (deq - x)^2 in double) against the
    oracle's float64 sums of the oracle's own quantization of the same x."""
    F = gpu_lib
    shape = (48, 80) if case == "nvfp4_ragged" else (256, 512)
    x = S.sparse_outliers(*shape, seed=11)
    xf = S.as_f32(x)
    if case == "mxfp4":
        q, _ = _gpu_quant(F, x, 1)
        ref = O.mxfp4_quantize(xf)
        want = O.quant_noise(xf, ref["codes"], ref["scales"], 1.0, block=(1, 32), e8m0=True)
    elif case == "nvfp4_2d":
        q, _ = _gpu_quant(F, x, 0, block=1)
        ref = O.nvfp4_quantize_2d(xf)
        want = O.quant_noise(xf, ref["codes"], ref["scales"], float(ref["s_dec"]), block=(16, 16))
    else:
        rnd = SR if case == "nvfp4_sr" else RTN
        q, _ = _gpu_quant(F, x, 0, round=rnd, seed=5, stream=1)
        ref = O.nvfp4_quantize_1d(xf, "sr" if rnd == SR else "rtn", sr_seed=5, sr_stream=1)
        want = O.quant_noise(xf, ref["codes"], ref["scales"], float(ref["s_dec"]))
    sums = torch.zeros(2, dtype=torch.float64, device="cuda")
    ws = F.Workspace()
    F.fp4_quant_noise(x.cuda(), q, sums, ws)
    torch.cuda.synchronize()
    got = sums.cpu().numpy()
    assert got[0] == pytest.approx(want[0], rel=1e-12)
    assert got[1] == pytest.approx(want[1], rel=1e-12)
    assert 0.0 < got[1] < got[0]


def test_edge_values(gpu_lib):
    F = gpu_lib
    rng = np.random.default_rng(0)
    cases = {
        "zeros": np.zeros((32, 64), np.float32),
        "neg_zero": -np.zeros((32, 64), np.float32),
        "subnormal_bf16": (rng.standard_normal((32, 64)) * 1e-39).astype(np.float32),
        "tiny_amax": (rng.standard_normal((32, 64)) * 1e-37).astype(np.float32),
        "huge": (rng.standard_normal((32, 64)) * 1e37).astype(np.float32),
        "one_hot": np.eye(32, 64, dtype=np.float32) * 3.0,
        "lattice": np.tile(np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -6, -4, -3, -2, -1.5, -1, -.5, -0.],
                                    np.float32), (32, 4)),
    }
    for name, arr in cases.items():
        x = S.to_bf16(arr)
        xf = S.as_f32(x)
        for rnd in (RTN, SR):
            q, qt = _gpu_quant(F, x, 0, round=rnd, round_t=rnd, seed=1, stream=1, stream_t=2, col=True)
            mode = "sr" if rnd else "rtn"
            _check_1d(q, O.nvfp4_quantize_1d(xf, mode, sr_seed=1, sr_stream=1), 0)
            _check_1d(qt, O.nvfp4_quantize_1d(np.ascontiguousarray(xf.T), mode, sr_seed=1,
                                              sr_stream=2), 0)
            qm, _ = _gpu_quant(F, x, 1, round=rnd, seed=1, stream=1)
            _check_1d(qm, O.mxfp4_quantize(xf, mode, sr_seed=1, sr_stream=1), 1)


def test_empty_tensor(gpu_lib):
    F = gpu_lib
    x = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")[:0]
    out = F.QTensor.empty(0, 64)
    F.fp4_quantize(x, out)
    torch.cuda.synchronize()
    assert float(out.amax.item()) == 0.0 and float(out.s_dec.item()) == 1.0


def test_supplied_amax(gpu_lib):
    F = gpu_lib
    x = S.normal((64, 128), 1.0, seed=4)
    q, qt = _gpu_quant(F, x, 0, amax_in=50.0, col=True)
    xf = S.as_f32(x)
    _check_1d(q, O.nvfp4_quantize_1d(xf, amax_in=50.0), 0)
    ref_t = O.nvfp4_quantize_1d(np.ascontiguousarray(xf.T))
    _check_1d(qt, ref_t, 0)           # the transposed output computes its own amax


def test_nonfinite_input_sets_status(gpu_lib):
    F = gpu_lib
    a = np.ones((32, 64), np.float32)
    a[3, 5] = np.inf
    x = S.to_bf16(a).cuda()
    out = F.QTensor.empty(32, 64)
    ws = F.Workspace()
    F.fp4_quantize(x, out, ws=ws)
    assert ws.status() == 7           # FP4_ERR_NONFINITE, recorded on the device
    ws.clear()
    assert ws.status() == 0


def test_llama_activation_sampled_rows(gpu_lib):
    """Full 32768 x 4096 activation (1% Student-t channels): quantized on the
    GPU in the bench's launch configuration; the oracle checks 64 sampled rows
    (with the full-tensor amax) of both the row-wise and transposed outputs."""
    F = gpu_lib
    M, K = 32768, 4096
    d = S.llama_linear(4096, K, M=M, seed=0)
    x = d["X"]
    q, qt = _gpu_quant(F, x, 0, round=RTN, round_t=SR, seed=0, stream_t=3, col=True)
    xf = S.as_f32(x)
    A = O.amax(xf)
    assert float(_np(q.amax)[0]) == A
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(M, 64, replace=False))
    codes = _np(q.codes).reshape(M, K // 2)
    for r in rows:
        ref = O.nvfp4_quantize_1d(xf[r:r + 1], amax_in=A, row_offset=int(r))
        assert np.array_equal(codes[r:r + 1], ref["codes"]), r
    kt = np.sort(rng.choice(K, 32, replace=False))
    codes_t = _np(qt.codes).reshape(K, M // 2)
    for k in kt:
        col = np.ascontiguousarray(xf[:, k][None, :])
        ref = O.nvfp4_quantize_1d(col, "sr", sr_seed=0, sr_stream=3, amax_in=A, row_offset=int(k))
        assert np.array_equal(codes_t[k:k + 1], ref["codes"]), k
