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
    r = lambda rnd: {0: "rtn", 1: "sr", 2: "quest"}[rnd]

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
        # W^T feeds dgrad: the QuEST-style forward scale does not apply there
        ops["wq_t"] = q1(T(W), 0 if cfg.round_fwd == 2 else cfg.round_fwd, rn if m & 2 else 0, 0)
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


@pytest.mark.parametrize("variant", ["nvfp4", "nvfp4_wgrad_rht", "nvfp4_1d_rht_all", "mxfp4",
                                     "mxfp4_quest"])
def test_tiny_linear_layer(gpu_lib, variant):
    F = gpu_lib
    d = S.tiny_linear(seed=0)
    fmt = 1 if variant.startswith("mxfp4") else 0
    cfg = F.linear_cfg(fmt, out_dtype=F.OUT_F32)
    if variant == "mxfp4_quest":
        cfg.round_fwd = F.QUEST           # Quartet: QuEST-style forward, RTN backward
    if variant == "nvfp4_wgrad_rht":
        cfg.rht_mask = F.RHT_WGRAD
    if variant == "nvfp4_1d_rht_all":
        # 1x16 weights, so that fprop and dgrad can rotate too: every operand
        # of the three GEMMs goes through the 16-point transform
        cfg.w_block = F.BLOCK_1D
        cfg.rht_mask = F.RHT_FPROP | F.RHT_DGRAD | F.RHT_WGRAD
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


# BF16 outputs: the FP32-accumulation bar plus at most 2^-9 relative rounding
# per element from the final BF16 store.
TOL_BF16 = TOL + 2.0 ** -9


@pytest.mark.parametrize("variant", ["nvfp4", "mxfp4"])
def test_llama_qkvo_layer_full_size_sampled(gpu_lib, variant):
    """One 7B QKVO layer (M = 32768 tokens, N = K = 4096) through
    fqt_linear_fwd / fqt_linear_bwd in the configuration the step benchmark
    times (BF16 Y and dX, FP32 dW).  The oracle checks W, W^T and X^T in full,
    32 sampled rows of X, dY and dY^T (with the full-tensor amax), and 32
    sampled rows of Y, dX and dW over the full contraction."""
    F = gpu_lib
    M, N, K = 32768, 4096, 4096
    nv = variant == "nvfp4"
    fmt, bs = (0, 16) if nv else (1, 32)
    d = S.llama_linear(N, K, M=M, seed=0)
    cfg = F.linear_cfg(fmt, out_dtype=F.OUT_BF16, seed=0)
    sv = F.Saved.empty(M, N, K, cfg, logical_scales=False)
    ws = F.Workspace(M, N, K)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    F.fqt_linear_fwd(cfg, d["X"].cuda(), d["W"].cuda(), y, sv, ws)
    F.fqt_linear_bwd(cfg, d["dY"].cuda(), sv, dx, dw, ws)
    torch.cuda.synchronize()
    assert ws.status() == 0

    X, W, dY = (S.as_f32(d[k]) for k in ("X", "W", "dY"))
    T = lambda a: np.ascontiguousarray(a.T)
    rn, m = cfg.rht_n, cfg.rht_mask
    rnd = lambda r: "sr" if r == 1 else "rtn"
    Ax, Ady = O.amax(X), O.amax(dY)

    def q1(a, r, rht, stream, amax_in=None, row_offset=0):
        if nv:
            return O.nvfp4_quantize_1d(a, rnd(r), rht_n=rht, rht_seed=0, sr_seed=0,
                                       sr_stream=stream, amax_in=amax_in, row_offset=row_offset)
        return O.mxfp4_quantize(a, rnd(r), rht_n=rht, rht_seed=0, sr_seed=0, sr_stream=stream,
                                row_offset=row_offset)

    def deq(q, blk=(1, 16)):
        return O.dequantize(q["codes"], q["scales"], blk if nv else (1, 32), not nv)

    def sel_rows(q, idx):
        return {"codes": q["codes"][idx], "scales": q["scales"][idx], "s_dec": q["s_dec"]}

    def got_codes(t, idx=None):
        c = t.codes.cpu().numpy().reshape(t.rows, t.cols // 2)
        return c if idx is None else c[idx]

    def got_scales(t):
        return from_mma_layout(t.scales_mma.cpu().numpy(), t.rows, t.cols // bs)

    def sampled(a, idx, r, rht, stream, A):
        """Rows idx of the quantization of a, one oracle call per row."""
        parts = [q1(a[i:i + 1], r, rht, stream, A, int(i)) for i in idx]
        return {"codes": np.concatenate([p["codes"] for p in parts]),
                "scales": np.concatenate([p["scales"] for p in parts]),
                "s_dec": parts[0]["s_dec"]}

    rng = np.random.default_rng(11)
    rows = np.sort(rng.choice(M, 32, replace=False))
    nsel = np.sort(rng.choice(N, 32, replace=False))

    # weights and X^T in full
    if nv:
        wq, wq_t, wblk = O.nvfp4_quantize_2d(W), O.nvfp4_quantize_2d(T(W)), (16, 16)
    else:
        wq = q1(W, cfg.round_fwd, rn if m & 1 else 0, 0)
        wq_t = q1(T(W), cfg.round_fwd, rn if m & 2 else 0, 0)
        wblk = (1, 32)
    xq_t = q1(T(X), cfg.round_x_t, rn if m & 4 else 0, 3)
    for name, t, ref in (("wq", sv.wq, wq), ("wq_t", sv.wq_t, wq_t), ("xq_t", sv.xq_t, xq_t)):
        assert np.array_equal(got_codes(t), ref["codes"]), name
        sc = expand_2d(ref["scales"], t.rows) if t.block == 1 else ref["scales"]
        assert np.array_equal(got_scales(t), sc), name
        assert float(t.s_dec.item()) == float(ref["s_dec"]), name

    # sampled rows of X, dY (row-wise) and dY^T
    xq = sampled(X, rows, cfg.round_fwd, rn if m & 1 else 0, 0, Ax)
    dyq = sampled(dY, rows, cfg.round_bwd, rn if m & 2 else 0, 1, Ady)
    dYt = T(dY[:, nsel])                                   # rows n of dY^T
    parts = [q1(dYt[j:j + 1], cfg.round_bwd, rn if m & 4 else 0, 2, Ady, int(n))
             for j, n in enumerate(nsel)]
    dyq_t = {"codes": np.concatenate([p["codes"] for p in parts]),
             "scales": np.concatenate([p["scales"] for p in parts]), "s_dec": parts[0]["s_dec"]}
    for name, t, ref, idx in (("xq", sv.xq, xq, rows), ("dyq", sv.dyq, dyq, rows),
                              ("dyq_t", sv.dyq_t, dyq_t, nsel)):
        assert np.array_equal(got_codes(t, idx), ref["codes"]), name
        assert np.array_equal(got_scales(t)[idx], ref["scales"]), name
        assert float(t.s_dec.item()) == float(ref["s_dec"]), name

    # outputs over the full contraction
    sd = lambda q: float(q["s_dec"])
    ry = O.gemm(deq(xq), deq(wq, wblk), s_dec_a=sd(xq), s_dec_b=sd(wq))
    rdx = O.gemm(deq(dyq), deq(wq_t, wblk), s_dec_a=sd(dyq), s_dec_b=sd(wq_t))
    rdw = O.gemm(deq(dyq_t), deq(xq_t), s_dec_a=sd(dyq_t), s_dec_b=sd(xq_t))
    ri, ni = torch.from_numpy(rows).cuda(), torch.from_numpy(nsel).cuda()
    assert rel_fro(y[ri].float().cpu().numpy(), ry) <= TOL_BF16
    assert rel_fro(dx[ri].float().cpu().numpy(), rdx) <= TOL_BF16
    assert rel_fro(dw[ni].cpu().numpy(), rdw) <= TOL
