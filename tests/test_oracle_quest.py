"""Pins for the oracle's QuEST-style MXFP4 forward quantizer ("Quartet",
Approach; Measured effects, ablations: the forward pass uses a QuEST-style
quantizer, Hadamard rotation then clipping).  The pages give no clipping
rule; the reading (the scale from alpha * RMS, alpha the Gaussian-MSE-optimal
clipping multiple of E2M1, through the OCP power-of-two rule) is pinned here
by the mathematics it rests on, not by the pages: "parity unpinned" against
the pages themselves."""
import numpy as np
from scipy import integrate, optimize, stats

import oracle as O

LEVELS = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])


def _gaussian_mse(alpha: float) -> float:
    """E[(x - q(x))^2] for x ~ N(0, 1), q = E2M1 round-to-nearest with the
    top level 6 at alpha (values beyond alpha clip), integrated cell by cell."""
    s = alpha / 6.0
    mids = (LEVELS[1:] + LEVELS[:-1]) / 2 * s
    edges = np.concatenate([[0.0], mids, [alpha, np.inf]])
    vals = np.concatenate([LEVELS * s, [6 * s]])
    tot = 0.0
    for lo, hi, v in zip(edges[:-1], edges[1:], vals):
        tot += integrate.quad(lambda x: (x - v) ** 2 * stats.norm.pdf(x), lo, hi,
                              epsabs=1e-14, epsrel=1e-12, limit=200)[0]
    return 2 * tot


def test_alpha_is_the_gaussian_mse_optimal_clipping_multiple():
    best = optimize.minimize_scalar(_gaussian_mse, bounds=(1.5, 6.0), method="bounded",
                                    options={"xatol": 1e-10}).x
    alpha = O.quest_alpha()
    assert abs(alpha - best) <= 1e-6 * best
    assert _gaussian_mse(alpha) < _gaussian_mse(0.98 * alpha)
    assert _gaussian_mse(alpha) < _gaussian_mse(1.02 * alpha)


def test_threshold_is_alpha_times_rms():
    rng = np.random.default_rng(1)
    for scale in (1e-3, 1.0, 37.0):
        b = (rng.standard_normal(32) * scale).astype(np.float32)
        exact = O.quest_alpha() * np.sqrt(np.mean(b.astype(np.float64) ** 2))
        assert abs(O.quest_threshold(b) - exact) <= 4e-7 * exact
    assert O.quest_threshold(np.ones(32, np.float32)) == np.float32(O.quest_alpha())
    assert O.quest_threshold(np.zeros(32, np.float32)) == 0.0
    # the mean square is over all 32 values, in order-fixed groups of 8
    b = np.zeros(32, np.float32)
    b[31] = 4.0
    assert O.quest_threshold(b) == np.float32(O.quest_alpha() * np.float32(np.sqrt(0.5)))


def test_scale_byte_follows_the_threshold():
    """Scale byte floor(log2 T) - 2 + 127, for thresholds across binades; a
    block of ones: T = alpha in [2, 4), scale 2^-1, every value encodes 2."""
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((64, 32)) * np.exp2(rng.integers(-20, 20, (64, 1)))).astype(np.float32)
    q = O.mxfp4_quantize(x, "quest")
    for r in range(64):
        t = O.quest_threshold(x[r])
        assert q["scales"][r, 0] == np.frexp(np.float64(t))[1] - 1 - 2 + 127
    ones = O.mxfp4_quantize(np.ones((1, 32), np.float32), "quest")
    assert ones["scales"][0, 0] == 126 and np.all(ones["codes"] == 0x44)
    zero = O.mxfp4_quantize(np.zeros((1, 32), np.float32), "quest")
    assert zero["scales"][0, 0] == 0 and np.all(zero["codes"] == 0)


def test_clipping_saturates_outliers_and_rounds_the_rest_to_nearest():
    x = np.full((1, 32), 0.75, np.float32)
    x[0, 9] = -40.0                       # T = alpha * rms(block) << 40
    q = O.mxfp4_quantize(x, "quest")
    e = int(q["scales"][0, 0]) - 127
    d = O.dequantize(q["codes"], q["scales"], (1, 32), True)[0]
    assert d[9] == -6.0 * 2.0 ** e        # clipped to the top level
    code = int(O.e2m1_rtn(np.float32(0.75 * 2.0 ** -e))[0])
    assert np.all(d[np.arange(32) != 9] == O.e2m1_value(code) * 2.0 ** e)
    rtn = O.mxfp4_quantize(x)             # the max rule keeps the outlier in range instead
    assert O.dequantize(rtn["codes"], rtn["scales"], (1, 32), True)[0, 9] < d[9]


def test_lower_error_than_max_scaling_on_rotated_gaussian_blocks():
    """On Hadamard-rotated Gaussian data the RMS-based scale gives a lower
    relative MSE than the block-max scale, near the Gaussian optimum
    (0.01268 for an ideal continuous scale)."""
    rng = np.random.default_rng(0)
    x = rng.standard_normal((512, 1024)).astype(np.float32)
    xr = O.rht_rows(x, 32, 3).astype(np.float64)
    err = {}
    for mode in ("rtn", "quest"):
        q = O.mxfp4_quantize(x, mode, rht_n=32, rht_seed=3)
        d = O.dequantize(q["codes"], q["scales"], (1, 32), True)
        err[mode] = np.mean((d - xr) ** 2) / np.mean(xr ** 2)
    assert err["quest"] < err["rtn"]
    assert abs(err["quest"] - _gaussian_mse(O.quest_alpha())) < 0.05 * err["quest"]
