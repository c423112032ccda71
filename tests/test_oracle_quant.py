"""Pins for the oracle's NVFP4 / MXFP4 quantizers and its GEMM reference.

What the pages fix ("FP4", How it works / Components / Hyperparameters):
16-value blocks with an E4M3 scale plus one FP32 tensor scale (NVFP4),
32-value blocks with a power-of-two E8M0 scale (MXFP4), values cast to the
E2M1 levels; two-dimensional quantization as a stabiliser.  The checks below
use brute force on tiny blocks, invariants that hold for any correct
implementation, special cases with closed forms, and exact rational GEMMs.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
from conftest import read_golden_numbers

LEVELS = [float(v) for v in read_golden_numbers("e2m1_levels.txt")]
FORMATS = {row[0]: row for row in
           np.array(read_golden_numbers("block_formats.txt")).reshape(-1, 4)}


def _codes(packed):
    lo = packed & 0xF
    hi = packed >> 4
    return np.stack([lo, hi], axis=-1).reshape(packed.shape[0], -1)


def _e2m1(codes):
    table = np.array([O.e2m1_value(c) for c in range(16)])
    return table[codes]


def test_block_sizes_follow_page():
    assert int(FORMATS["NVFP4"][1]) == 16 and FORMATS["NVFP4"][2] == "E4M3"
    assert int(FORMATS["MXFP4"][1]) == 32 and FORMATS["MXFP4"][2] == "E8M0"
    x = np.random.default_rng(0).standard_normal((2, 64)).astype(np.float32)
    assert O.nvfp4_quantize_1d(x)["scales"].shape == (2, 64 // 16)
    assert O.mxfp4_quantize(x)["scales"].shape == (2, 64 // 32)


def _tiny_blocks(rng, n):
    xs = []
    for i in range(n):
        scale = 10.0 ** rng.uniform(-6, 4)
        x = rng.standard_normal(16) * scale
        if i % 5 == 0:
            x[rng.integers(16)] *= 50.0            # one outlier
        if i % 7 == 0:
            x[:8] = 0.0                             # half block of zeros
        xs.append(x)
    return np.array(xs, np.float32)


def test_nvfp4_bruteforce_tiny_blocks():
    """Per block: sf is E4M3(b * s_enc / 6); each code is the argmin over all
    16 codes of |x * inv - e2m1(c)| (ties: even code); the block max maps to
    +-6 when sf is normal; reconstruction error within half a level gap."""
    rng = np.random.default_rng(11)
    X = _tiny_blocks(rng, 400)
    q = O.nvfp4_quantize_1d(X.reshape(1, -1))
    A = np.float32(np.abs(X).max())
    assert q["amax"] == A
    s_enc, s_dec = O.nvfp4_global_scales(A)
    assert s_enc == np.float32(2688.0) / A and s_dec == A / np.float32(2688.0)
    codes = _codes(q["codes"]).reshape(-1, 16)
    scales = q["scales"].reshape(-1)
    allv = np.array([O.e2m1_value(c) for c in range(16)])
    for blk in range(X.shape[0]):
        x = X[blk]
        b = np.float32(np.abs(x).max())
        t = np.float32(np.float32(b * s_enc) / np.float32(6.0))
        sf = int(scales[blk])
        assert sf == int(O.e4m3_rne_sat([t])[0])
        sfv = np.float32(O.e4m3_value(sf))
        inv = np.float32(0.0) if sf == 0 else np.float32(s_enc / sfv)
        v = (x * inv).astype(np.float32)
        for j in range(16):
            d = np.abs(float(v[j]) - allv)
            best = np.flatnonzero(d == d.min())
            cands = [c for c in best if (c & 8) == (8 if np.signbit(v[j]) else 0) or allv[c] != 0]
            want = min(cands, key=lambda c: (c & 1, c & 8 != (8 if np.signbit(v[j]) else 0)))
            assert _e2m1(codes[blk, j]) == allv[want], (blk, j, v[j], codes[blk, j], want)
        if sf >= 0x08 and sf < 0x7E and b > 0:     # normal, unsaturated scale
            jm = int(np.argmax(np.abs(x)))
            assert abs(_e2m1(codes[blk, jm])) == 6.0
        xhat = _e2m1(codes[blk]) * O.e4m3_value(sf) * float(s_dec)
        if sf == 0:
            # the block scale underflows E4M3 (t at most half the smallest
            # subnormal, 2^-10): the whole block flushes to zero
            assert float(t) <= 2.0 ** -10 and not xhat.any()
            continue
        gap = 2.0 * O.e4m3_value(sf) * float(s_dec)   # largest level gap is 2
        sat = np.abs(v) > 6.0                          # saturated elements code +-6
        assert np.all(np.abs(_e2m1(codes[blk][sat])) == 6.0)
        assert np.all(np.abs(xhat - x)[~sat] <= 0.5 * gap * (1 + 1e-6) + 1e-30)


def test_nvfp4_special_cases():
    # all-zero tensor: s_dec = s_enc = 1, zero scales and codes; -0 keeps its sign
    z = np.zeros((2, 32), np.float32)
    z[1, 3] = -0.0
    q = O.nvfp4_quantize_1d(z)
    assert q["amax"] == 0 and q["s_dec"] == 1.0
    assert not q["scales"].any()
    assert _codes(q["codes"])[1, 3] == 8 and _codes(q["codes"])[0].sum() == 0
    # the block holding the tensor max gets the top scale 448 (0x7E)
    rng = np.random.default_rng(12)
    x = rng.standard_normal((8, 64)).astype(np.float32)
    x[5, 17] = 40.0
    q = O.nvfp4_quantize_1d(x)
    assert q["scales"][5, 1] == 0x7E
    assert _codes(q["codes"])[5, 17] == 7
    # a supplied amax is used as given
    q2 = O.nvfp4_quantize_1d(x, amax_in=80.0)
    assert q2["amax"] == np.float32(80.0) and q2["scales"][5, 1] < 0x7E
    # a block whose scale underflows E4M3 (b * s_enc / 6 below 2^-10) has
    # scale code 0 and encodes to zeros, keeping only the signs
    y = np.zeros((1, 32), np.float32)
    y[0, 0] = 1.0e6                       # s_enc = 2688 / 1e6
    y[0, 16:] = np.linspace(-1.0, 1.0, 16, dtype=np.float32)
    q3 = O.nvfp4_quantize_1d(y)
    assert q3["scales"][0, 1] == 0
    assert np.all(_codes(q3["codes"])[0, 16:] & 7 == 0)


def test_nvfp4_row_offset_and_sr_index():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((12, 64)).astype(np.float32)
    full = O.nvfp4_quantize_1d(x, "sr", sr_seed=3, sr_stream=2)
    part = O.nvfp4_quantize_1d(x[5:9], "sr", sr_seed=3, sr_stream=2, amax_in=full["amax"],
                               row_offset=5)
    assert np.array_equal(part["codes"], full["codes"][5:9])
    assert np.array_equal(part["scales"], full["scales"][5:9])
    # the draw index follows the row-major logical layout: identical rows get
    # different stochastic codes somewhere
    y = np.tile(x[:1], (4, 1))
    q = O.nvfp4_quantize_1d(y, "sr", sr_seed=3, sr_stream=2)
    assert not np.array_equal(q["codes"][0], q["codes"][1])
    # stochastic rounding reproduces RTN on values that sit on the lattice
    lat = np.array([LEVELS * 8], np.float32)[:, :64]
    assert np.array_equal(O.nvfp4_quantize_1d(lat, "sr", sr_seed=9)["codes"],
                          O.nvfp4_quantize_1d(lat)["codes"])


def _unit_scale_blocks(rng, R, C, bs):
    """x[R, C] whose every bs-block has max |x| = 6 exactly and whose other
    values are arbitrary binary32 numbers in (-6, 6): with a tensor amax of
    2688 (NVFP4: s_enc = 1, block scale E4M3(1) = 1) or directly (MXFP4:
    scale 2^(floor(log2 6) - 2) = 1) every value reaches E2M1 rounding
    unscaled."""
    x = rng.uniform(-6.0, 6.0, (R, C)).astype(np.float32)
    x[:, ::bs] = np.where(rng.random((R, C // bs)) < 0.5, -6.0, 6.0)
    return x


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_sr_draw_index_is_row_major_in_the_operand(fmt):
    """Element (r, c) of rows starting at row_offset of an [*, C] operand is
    rounded with draw (row_offset + r) * C + c of its stream (the layout
    reading), checked value by value where the scales are exactly 1."""
    rng = np.random.default_rng(31)
    R, C, off, seed, stream = 3, 64, 5, 11, 2
    bs = 16 if fmt == "nvfp4" else 32
    x = _unit_scale_blocks(rng, R, C, bs)
    if fmt == "nvfp4":
        q = O.nvfp4_quantize_1d(x, "sr", sr_seed=seed, sr_stream=stream, amax_in=2688.0,
                                row_offset=off)
        assert np.all(q["scales"] == O.e4m3_rne_sat(np.float32(1.0))[0])
    else:
        q = O.mxfp4_quantize(x, "sr", sr_seed=seed, sr_stream=stream, row_offset=off)
        assert np.all(q["scales"] == 127)
    u = O.draws16(seed, stream, off * C, R * C).reshape(R, C)
    want = O.e2m1_sr(x.reshape(-1), u.reshape(-1)).reshape(R, C)
    assert np.array_equal(_codes(q["codes"]), want)


def test_amax_is_of_magnitudes():
    """The tensor amax is max |x|: a tensor whose extreme is negative."""
    x = np.array([[-5.0, 1.0, 2.0, -0.5] * 4], np.float32)
    assert O.amax(x) == 5.0
    assert O.nvfp4_quantize_1d(x)["amax"] == 5.0
    assert O.nvfp4_quantize_2d(np.tile(x, (16, 1)))["amax"] == 5.0
    y = np.random.default_rng(32).standard_normal((8, 32)).astype(np.float32)
    y[3, 9] = -40.0
    assert O.amax(y) == 40.0


def test_nvfp4_rht_amax_is_of_rotated_tensor():
    rng = np.random.default_rng(14)
    x = rng.standard_normal((4, 64)).astype(np.float32)
    x[2, 7] = 30.0
    q = O.nvfp4_quantize_1d(x, rht_n=16, rht_seed=21)
    xr = O.rht_rows(x, 16, 21)
    assert q["amax"] == np.float32(np.abs(xr).max())
    assert q["amax"] < 30.0          # the outlier is spread over its block
    plain = O.nvfp4_quantize_1d(xr)
    assert np.array_equal(plain["codes"], q["codes"])


def test_nvfp4_2d_tile_scale_and_transpose():
    rng = np.random.default_rng(15)
    w = (rng.standard_normal((48, 64)) * 0.02).astype(np.float32)
    w[17, 33] = 0.5
    q = O.nvfp4_quantize_2d(w)
    qt = O.nvfp4_quantize_2d(np.ascontiguousarray(w.T))
    assert q["amax"] == qt["amax"] == np.float32(0.5)
    assert np.array_equal(qt["scales"], q["scales"].T)
    assert np.array_equal(_codes(qt["codes"]), _codes(q["codes"]).T)
    assert q["scales"][1, 2] == 0x7E
    # one scale per 16x16 tile: the tile scale equals a 1-D quantization of
    # the flattened tile with the same tensor amax
    s_enc, _ = O.nvfp4_global_scales(q["amax"])
    codes = _codes(q["codes"])
    for i in range(3):
        for j in range(4):
            tile = w[16 * i:16 * i + 16, 16 * j:16 * j + 16]
            t = np.float32(np.float32(np.abs(tile).max() * s_enc) / np.float32(6.0))
            assert q["scales"][i, j] == O.e4m3_rne_sat([t])[0], (i, j)
            # the tile's largest magnitude lands on the top level, 6
            a, b = np.unravel_index(np.argmax(np.abs(tile)), tile.shape)
            assert abs(O.e2m1_value(int(codes[16 * i + a, 16 * j + b]))) == 6.0, (i, j)


def test_mxfp4_scale_rule_and_bounds():
    rng = np.random.default_rng(16)
    x = (rng.standard_normal((16, 128)) * 10.0 ** rng.uniform(-5, 5, (16, 1))).astype(np.float32)
    x[3, :32] = 0.0
    q = O.mxfp4_quantize(x)
    codes = _codes(q["codes"])
    for r in range(16):
        for b in range(4):
            blk = x[r, b * 32:(b + 1) * 32]
            bmax = float(np.abs(blk).max())
            s = int(q["scales"][r, b])
            if bmax == 0:
                assert s == 0 and not (codes[r, b * 32:(b + 1) * 32] & 7).any()
                continue
            e = int(np.floor(np.log2(bmax))) - 2
            assert s == e + 127
            v = blk / 2.0 ** e
            assert np.all(np.abs(v) < 8)
            deq = _e2m1(codes[r, b * 32:(b + 1) * 32]) * 2.0 ** e
            assert np.all(np.abs(deq - blk) <= 2.0 ** (e + 1) + 1e-30)
            jm = int(np.argmax(np.abs(blk)))
            assert abs(_e2m1(codes[r, b * 32 + jm])) in (4.0, 6.0)


def test_nvfp4_error_below_mxfp4():
    """NVFP4's smaller block and finer scale give lower quantization error
    ("FP4", Components, NVFP4) -- a trend check on Gaussian data."""
    rng = np.random.default_rng(17)
    x = rng.standard_normal((64, 256)).astype(np.float32)
    qn = O.nvfp4_quantize_1d(x)
    qm = O.mxfp4_quantize(x)
    xn = O.dequantize(qn["codes"], qn["scales"]) * float(qn["s_dec"])
    xm = O.dequantize(qm["codes"], qm["scales"], block=(1, 32), e8m0=True)
    en = np.mean((xn - x) ** 2) / np.mean(x ** 2)
    em = np.mean((xm - x) ** 2) / np.mean(x ** 2)
    assert en < em


def _fraction_gemm(ac, asc, bc, bsc, block):
    """Exact rational GEMM from the page's level table (independent decode)."""
    lv = [Fraction(v) for v in LEVELS]

    def val(code):
        m = lv[code & 7]
        return -m if code & 8 else m

    def e4m3(s):
        e, m = (s >> 3) & 15, s & 7
        return Fraction(m, 8) * Fraction(1, 64) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)

    M, K = ac.shape
    N = bc.shape[0]
    out = np.zeros((M, N), dtype=object)
    for i in range(M):
        for j in range(N):
            s = Fraction(0)
            for k in range(K):
                s += (val(int(ac[i, k])) * e4m3(int(asc[i // block[0], k // block[1]])) *
                      val(int(bc[j, k])) * e4m3(int(bsc[j // block[0], k // block[1]])))
            out[i, j] = s
    return out


def test_gemm_reference_exact_on_small_case():
    rng = np.random.default_rng(18)
    A = rng.standard_normal((4, 32)).astype(np.float32)
    B = rng.standard_normal((3, 32)).astype(np.float32)
    qa = O.nvfp4_quantize_1d(A)
    qb = O.nvfp4_quantize_1d(B)
    ah = O.dequantize(qa["codes"], qa["scales"])
    bh = O.dequantize(qb["codes"], qb["scales"])
    got = O.gemm(ah, bh)
    ref = _fraction_gemm(_codes(qa["codes"]), qa["scales"], _codes(qb["codes"]), qb["scales"], (1, 16))
    assert all(got[i, j] == float(ref[i, j]) for i in range(4) for j in range(3))
    scaled = O.gemm(ah, bh, alpha=2.0, s_dec_a=qa["s_dec"], s_dec_b=qb["s_dec"])
    assert np.allclose(scaled, got * 2.0 * float(qa["s_dec"]) * float(qb["s_dec"]), rtol=1e-15)


def test_gemm_one_hot_selects_entries():
    # K = 16, a single block: one-hot rows of A pick single columns of B
    B = np.random.default_rng(19).standard_normal((5, 16)).astype(np.float32)
    qb = O.nvfp4_quantize_1d(B)
    bh = O.dequantize(qb["codes"], qb["scales"])
    A = np.zeros((16, 16), np.float32)
    A[np.arange(16), np.arange(16)] = 6.0
    qa = O.nvfp4_quantize_1d(A)
    ah = O.dequantize(qa["codes"], qa["scales"])
    assert np.array_equal(ah, np.eye(16) * ah[0, 0])
    got = O.gemm(ah, bh)
    assert np.array_equal(got, ah[0, 0] * bh.T)


def test_gemm_of_quantized_close_to_unquantized():
    rng = np.random.default_rng(20)
    X = rng.standard_normal((64, 512)).astype(np.float32)
    W = (rng.standard_normal((32, 512)) * 0.02).astype(np.float32)
    qx, qw = O.nvfp4_quantize_1d(X), O.nvfp4_quantize_2d(W)
    y = O.gemm(O.dequantize(qx["codes"], qx["scales"]),
               O.dequantize(qw["codes"], qw["scales"], block=(16, 16)),
               s_dec_a=qx["s_dec"], s_dec_b=qw["s_dec"])
    ref = X.astype(np.float64) @ W.T.astype(np.float64)
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert 0.02 < rel < 0.2      # FP4 noise level, not a gross mistake


def test_nvfp4_reciprocal_saturates_for_subnormal_blocks():
    """reading: when s_enc / sf overflows (only a block whose max is below
    ~1.8e-38 can cause it) the reciprocal is the largest finite float, so a
    zero stays a zero and nothing becomes NaN or saturates spuriously."""
    rng = np.random.default_rng(21)
    x = (rng.standard_normal((4, 64)) * 1e-39).astype(np.float32)
    x[0, :8] = 0.0
    x[1, :4] = -0.0
    q = O.nvfp4_quantize_1d(x)
    codes = _codes(q["codes"])
    assert (codes[0, :8] == 0).all() and (codes[1, :4] == 8).all()
    s_enc, _ = O.nvfp4_global_scales(q["amax"])
    assert s_enc == np.float32(3.4028235e38)          # 2688 / amax overflowed
    v = _e2m1(codes)
    assert np.isfinite(v).all() and (np.abs(v) <= 6).all()
    assert (np.sign(v[v != 0]) == np.sign(x[v != 0])).all()


def test_quant_noise_closed_form_mxfp4_block():
    """One MXFP4 block [4, 0.25, 1.25, 0, ...]: the block scale is 2^0 (max 4,
    floor(log2 4) - 2 = 0); 0.25 and 1.25 are midpoints that round to the
    even levels 0 and 1, each off by 0.25.  sum x^2 = 16 + 1/16 + 25/16,
    sum noise^2 = 2/16."""
    x = np.zeros((1, 32), np.float32)
    x[0, :3] = [4.0, 0.25, 1.25]
    q = O.mxfp4_quantize(x)
    sx, sn = O.quant_noise(x, q["codes"], q["scales"], 1.0, block=(1, 32), e8m0=True)
    assert sx == 17.625
    assert sn == 0.125


def test_quant_noise_zero_for_representable_blocks():
    """Values already on the E2M1 grid of their block scale carry no noise."""
    x = np.zeros((2, 32), np.float32)
    x[0, :8] = [6, 4, 3, 2, 1.5, 1, 0.5, 0]
    x[1, :8] = [-6, -3, -1, -0.5, 0.5, 1, 2, 4]
    q = O.mxfp4_quantize(x)
    sx, sn = O.quant_noise(x, q["codes"], q["scales"], 1.0, block=(1, 32), e8m0=True)
    assert sn == 0.0
    assert sx == float(np.sum(x.astype(np.float64) ** 2))


def test_quant_noise_matches_independent_decode_nvfp4():
    """NVFP4 with a tensor scale: the noise sum equals the one computed from
    an independent decode (E2M1 levels from the page's level set, E4M3 block
    scales through ml_dtypes) and is below the bound of half a level gap
    (at most 1 in units of the block scale) per element."""
    ml_dtypes = pytest.importorskip("ml_dtypes")
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((8, 64)) * np.exp(rng.uniform(-3, 3, (8, 1)))).astype(np.float32)
    q = O.nvfp4_quantize_1d(x)
    sx, sn = O.quant_noise(x, q["codes"], q["scales"], float(q["s_dec"]))
    codes = _codes(q["codes"])
    vals = np.where(codes >= 8, -np.array(LEVELS)[codes & 7], np.array(LEVELS)[codes & 7])
    sc = q["scales"].view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    deq = vals * np.repeat(sc, 16, axis=1) * float(q["s_dec"])
    d = deq - x.astype(np.float64)
    assert sx == pytest.approx(float(np.sum(x.astype(np.float64) ** 2)), rel=1e-15)
    assert sn == pytest.approx(float(np.sum(d * d)), rel=1e-15)
    gap_bound = np.repeat(sc, 16, axis=1) * float(q["s_dec"])      # half of the widest gap (2)
    assert np.all(np.abs(d) <= gap_bound * (1 + 1e-6))
