"""The fully quantized linear layer (fqt_linear_fwd / fqt_linear_bwd) vs the
oracle composed step by step: quantized operands bit-exact, Y, dX and dW
within a relative Frobenius error of 1e-3 of the float64 GEMMs.

NVFP4 mode follows "FP4 All the Way" (round-to-nearest forward, stochastic
rounding for the backward and update passes; 16x16 weight tiles); MXFP4 mode
follows "Quartet" (round-to-nearest backward, 32-point block Hadamard on the
operands of all three GEMMs).
"""
import numpy as np
import pytest
import torch

import fqt_synth as S
import oracle as O
from fp4_testlib import expand_2d, from_mma_layout, rel_fro

pytestmark = pytest.mark.gpu
TOL = 1e-3


def _oracle_layer(X, W, dY, cfg):
    """The layer's quantized operands and GEMMs, from the oracle only."""
    nv = cfg.fmt == 0
    T = lambda a: np.ascontiguousarray(a.T)
    rn, seed, m = cfg.rht_n, cfg.seed, cfg.rht_mask
    r = lambda rnd: "sr" if rnd == 1 else "rtn"

    def q1(a, rnd, rht, stream):
        if nv:
            return O.nvfp4_quantize_1d(a, r(rnd), rht_n=rht, rht_seed=seed, sr_seed=seed,
                                       sr_stream=stream)
        return O.mxfp4_quantize(a, r(rnd), rht_n=rht, rht_seed=seed, sr_seed=seed,
                                sr_stream=stream)

    def deq(q, blk=(1, 16)):
        if nv:
            return O.dequantize(q["codes"], q["scales"], blk) * float(q["s_dec"])
        return O.dequantize(q["codes"], q["scales"], (1, 32), True)

    ops = {}
    ops["xq"] = q1(X, cfg.round_fwd, rn if m & 1 else 0, 0)
    ops["xq_t"] = q1(T(X), cfg.round_x_t, rn if m & 4 else 0, 3)
    if nv and cfg.w_block == 1:
        ops["wq"], ops["wq_t"] = O.nvfp4_quantize_2d(W), O.nvfp4_quantize_2d(T(W))
        wblk = (16, 16)
    else:
        ops["wq"] = q1(W, cfg.round_fwd, rn if m & 1 else 0, 0)
        ops["wq_t"] = q1(T(W), cfg.round_fwd, rn if m & 2 else 0, 0)
        wblk = (1, 16)
    ops["dyq"] = q1(dY, cfg.round_bwd, rn if m & 2 else 0, 1)
    ops["dyq_t"] = q1(T(dY), cfg.round_bwd, rn if m & 4 else 0, 2)
    y = deq(ops["xq"]) @ deq(ops["wq"], wblk).T
    dx = deq(ops["dyq"]) @ deq(ops["wq_t"], wblk).T
    dw = deq(ops["dyq_t"]) @ deq(ops["xq_t"]).T
    return ops, y, dx, dw


def _run_layer(F, X, W, dY, cfg):
    M, K = X.shape
    N = W.shape[0]
    sv = F.Saved.empty(M, N, K, cfg, logical_scales=False)
    ws = F.Workspace(M, N, K)
    y = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    dx = torch.zeros((M, K), dtype=torch.float32, device="cuda")
    dw = torch.zeros((N, K), dtype=torch.float32, device="cuda")
    F.fqt_linear_fwd(cfg, X.cuda(), W.cuda(), y, sv, ws)
    F.fqt_linear_bwd(cfg, dY.cuda(), sv, dx, dw, ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    return sv, y.cpu().numpy(), dx.cpu().numpy(), dw.cpu().numpy()


def _compare_ops(F, sv, ops, cfg):
    bs = 16 if cfg.fmt == 0 else 32
    for name in ("xq", "xq_t", "wq", "wq_t", "dyq", "dyq_t"):
        t, ref = getattr(sv, name), ops[name]
        codes = t.codes.cpu().numpy().reshape(t.rows, t.cols // 2)
        assert np.array_equal(codes, ref["codes"]), name
        per_row = ref["scales"]
        if t.block == 1:
            per_row = expand_2d(per_row, t.rows)
        got = from_mma_layout(t.scales_mma.cpu().numpy(), t.rows, t.cols // bs)
        assert np.array_equal(got, per_row), name
        assert float(t.s_dec.item()) == float(ref["s_dec"]), name


@pytest.mark.parametrize("variant", ["nvfp4", "nvfp4_wgrad_rht", "mxfp4"])
def test_tiny_linear_layer(gpu_lib, variant):
    F = gpu_lib
    d = S.tiny_linear(seed=0)
    fmt = 1 if variant == "mxfp4" else 0
    cfg = F.linear_cfg(fmt, out_dtype=F.OUT_F32)
    if variant == "nvfp4_wgrad_rht":
        cfg.rht_mask = F.RHT_WGRAD
    X, W, dY = d["X"], d["W"], d["dY"]
    sv, y, dx, dw = _run_layer(F, X, W, dY, cfg)
    ops, ry, rdx, rdw = _oracle_layer(S.as_f32(X), S.as_f32(W), S.as_f32(dY), cfg)
    _compare_ops(F, sv, ops, cfg)
    for got, ref, name in ((y, ry, "Y"), (dx, rdx, "dX"), (dw, rdw, "dW")):
        err = rel_fro(got, ref)
        assert err <= TOL, (name, err)


def test_linear_ragged_sizes(gpu_lib):
    """M, N, K multiples of 128 but not of the 256-wide N tile or of the
    256-element K stage."""
    F = gpu_lib
    M, N, K = 384, 640, 384
    X = S.sparse_outliers(M, K, seed=1)
    W = S.normal((N, K), 0.02, seed=2)
    dY = S.normal((M, N), 1e-3, seed=3)
    cfg = F.linear_cfg(0, out_dtype=F.OUT_F32, seed=77)
    sv, y, dx, dw = _run_layer(F, X, W, dY, cfg)
    ops, ry, rdx, rdw = _oracle_layer(S.as_f32(X), S.as_f32(W), S.as_f32(dY), cfg)
    _compare_ops(F, sv, ops, cfg)
    for got, ref in ((y, ry), (dx, rdx), (dw, rdw)):
        assert rel_fro(got, ref) <= TOL


def test_linear_quantized_result_tracks_unquantized(gpu_lib):
    """Sanity: the FP4 layer stays within FP4 noise of the unquantized one."""
    F = gpu_lib
    d = S.tiny_linear(seed=0)
    cfg = F.linear_cfg(0, out_dtype=F.OUT_F32)
    _, y, dx, dw = _run_layer(F, d["X"], d["W"], d["dY"], cfg)
    X, W, dY = (S.as_f32(d[k]).astype(np.float64) for k in ("X", "W", "dY"))
    assert rel_fro(y, X @ W.T) < 0.2
    assert rel_fro(dx, dY @ W) < 0.3
    assert rel_fro(dw, dY.T @ X) < 0.3
