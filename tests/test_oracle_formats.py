"""Pins for the oracle's number formats (E2M1, E4M3, E8M0).

Each check compares the oracle with something other than itself: the level
set printed on the "FP4" page (Components, "E2M1 format"), known values of
the formats, or the conversion routines of the ml_dtypes library.
"""
import math

import ml_dtypes as md
import numpy as np
import pytest

import oracle as O
from conftest import read_golden_numbers


def _all_bf16_finite() -> np.ndarray:
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    return f[np.isfinite(f)]


def test_e2m1_levels_match_page():
    levels = [float(v) for v in read_golden_numbers("e2m1_levels.txt")]
    assert len(levels) == 8
    got = [O.e2m1_value(c) for c in range(8)]
    assert got == levels
    # sign bit (bit 3) negates; -0 is code 8
    for c in range(8):
        assert O.e2m1_value(c | 8) == -levels[c]
    assert math.copysign(1.0, O.e2m1_value(8)) == -1.0


def test_e2m1_rtn_matches_ml_dtypes_on_every_bf16():
    x = _all_bf16_finite()
    ours = O.e2m1_rtn(x)
    ref = x.astype(md.float4_e2m1fn).view(np.uint8) & 0xF
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first x={x[bad[:5]]} ours={ours[bad[:5]]} ref={ref[bad[:5]]}"


def test_e2m1_rtn_threshold_form():
    """Independent formulation: count the decision thresholds (midpoints of
    the page's level set) that |v| lies above; at a midpoint the level with
    the even code wins."""
    levels = [float(v) for v in read_golden_numbers("e2m1_levels.txt")]
    mids = [(levels[i] + levels[i + 1]) / 2 for i in range(7)]
    pts = [0.0, 7.0, 100.0, 1e-30]
    for m in mids:
        m32 = np.float32(m)
        pts += [m, float(np.nextafter(m32, np.float32(0))), float(np.nextafter(m32, np.float32(10)))]
    pts += list(np.random.default_rng(1).uniform(0, 8, 4000))
    v = np.array(pts + [-p for p in pts], np.float32)
    ours = O.e2m1_rtn(v)
    for vi, code in zip(v, ours):
        a = abs(float(vi))
        k = 0
        for i, m in enumerate(mids):
            if a > m or (a == m and (i + 1) % 2 == 0):
                k = i + 1
        want = k | (8 if math.copysign(1.0, float(vi)) < 0 else 0)
        assert code == want, (vi, code, want)


def test_e4m3_decode_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = codes.view(md.float8_e4m3fn).astype(np.float64)
    ours = np.array([O.e4m3_value(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_known_values():
    assert O.e4m3_value(0x7E) == 448.0          # largest finite
    assert O.e4m3_value(0x01) == 2.0 ** -9      # smallest subnormal
    assert O.e4m3_value(0x08) == 2.0 ** -6      # smallest normal
    assert O.e4m3_value(0x38) == 1.0
    assert O.e4m3_rne_sat([448.0, 1e6, 3.4e38])[0] == 0x7E
    assert list(O.e4m3_rne_sat([448.0, 1e6, 3.4e38])) == [0x7E] * 3
    assert list(O.e4m3_rne_sat([0.0, 2.0 ** -10, 2.0 ** -10 * 1.001])) == [0, 0, 1]


def test_e4m3_encode_matches_ml_dtypes():
    vals = [O.e4m3_value(c) for c in range(0x7F)]
    pts = []
    for i in range(len(vals)):
        v = np.float32(vals[i])
        pts += [v, np.nextafter(v, np.float32(0)), np.nextafter(v, np.float32(1e9))]
        if i + 1 < len(vals):
            m = np.float32((vals[i] + vals[i + 1]) / 2)
            pts += [m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(1e9))]
    rng = np.random.default_rng(2)
    pts += list(np.exp2(rng.uniform(-14, np.log2(448.0), 200_000)).astype(np.float32))
    t = np.array(pts, np.float32)
    t = t[(t >= 0) & (t <= 448.0)]
    ours = O.e4m3_rne_sat(t)
    ref = t.astype(md.float8_e4m3fn).view(np.uint8)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, (t[bad[:5]], ours[bad[:5]], ref[bad[:5]])
    # above the largest finite value the encoder saturates (satfinite)
    big = np.array([448.5, 463.9, 464.0, 480.0, 1e30], np.float32)
    assert (O.e4m3_rne_sat(big) == 0x7E).all()


def test_e8m0_decode_and_floor_log2():
    codes = np.arange(256, dtype=np.uint8)
    ref = codes.view(md.float8_e8m0fnu).astype(np.float64)
    ours = np.array([O.e8m0_value(int(c)) for c in codes])
    assert np.isnan(ours[255]) and np.isnan(ref[255])
    assert np.array_equal(ours[:255], ref[:255])
    rng = np.random.default_rng(3)
    bits = rng.integers(1, 0x7F800000, 100_000, dtype=np.uint64).astype(np.uint32)
    xs = bits.view(np.float32)
    for x in list(xs[:20000]) + [np.float32(1.0), np.float32(2.0 ** -149), np.float32(2.0 ** -127),
                                 np.float32(3.4e38), np.float32(0.75)]:
        m, e = math.frexp(float(x))          # x = m * 2^e, 0.5 <= m < 1
        assert O.floor_log2(x) == e - 1, x


@pytest.mark.parametrize("v", [0.0, 0.5, 3.0, 6.0, -1.5, -4.0])
def test_e2m1_lattice_is_fixed_by_rtn(v):
    code = int(O.e2m1_rtn([v])[0])
    assert O.e2m1_value(code) == v
