"""Pins for the oracle's stochastic rounding and its Philox4x32-10 draws.

Stochastic rounding ("FP4 All the Way", Key points: stochastic rounding for
the backward and update passes) is pinned by what the definition of an
unbiased stochastic rounding fixes: lattice points are fixed, the rounding
is unbiased (mean over 4096 seeds within 3 sigma; exactly, over all 2^16
draws, for values whose gap fraction has at most 16 bits), the up-probability
is the fraction of the gap to 16 bits, and for a fixed draw the result is
monotone in v.
Philox is pinned block for block against an independent Philox4x32-10
(cuRAND's host generator, which runs on the CPU), statistically (uniformity,
bit balance, independence of streams) and by its counter structure.
"""
import numpy as np

import oracle as O
from conftest import read_golden_numbers

LEVELS = [float(v) for v in read_golden_numbers("e2m1_levels.txt")]


def _val(codes):
    return np.array([O.e2m1_value(int(c)) for c in codes])


def test_lattice_points_fixed_for_any_draw():
    u = np.arange(0, 65536, 1024, dtype=np.uint32).astype(np.uint16)
    u = np.concatenate([u, np.array([1, 65535], np.uint16)])
    for lv in LEVELS:
        for s in (1.0, -1.0):
            v = np.full(u.size, s * lv, np.float32)
            out = _val(O.e2m1_sr(v, u))
            assert np.all(out == s * lv)


def _up_count(v: float) -> int:
    """How many of the 2^16 possible draws round |v| up (exhaustive)."""
    u = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    out = np.abs(_val(O.e2m1_sr(np.full(65536, v, np.float32), u)))
    a = min(abs(float(v)), 6.0)
    lo = max(l for l in LEVELS if l <= a)
    hi = min(l for l in LEVELS if l >= a)
    assert np.all((out == lo) | (out == hi))
    return int((out == hi).sum()) if hi != lo else 0


def test_exact_up_probability_on_the_16_bit_grid():
    """Over all 2^16 draws, a value whose gap fraction p has at most 16 bits
    rounds up exactly p * 2^16 times: the rounding is exactly unbiased there
    (mean = v), at every gap size and both signs."""
    cases = [(1.25, 0.5), (2.25, 0.25), (5.5, 0.75), (0.3125, 0.625), (-3.875, 0.875),
             (1.0 + 2.0 ** -17, 2.0 ** -16), (4.0 + 2.0 ** -15, 2.0 ** -16), (-0.5 - 2.0 ** -17, 2.0 ** -16),
             (5.999969482421875, 1.0 - 2.0 ** -16)]
    for v, p in cases:
        assert _up_count(v) == round(p * 65536), (v, p)


def test_up_probability_is_p_truncated_to_16_bits():
    """For any p the up-count lies in (p * 2^16 - 1, p * 2^16]: the bias is
    below 2^-16 of the gap and towards the lower level; p below 2^-16 never
    rounds up; beyond 6 saturates."""
    rng = np.random.default_rng(3)
    vals = np.concatenate([rng.uniform(-6, 6, 48), [2.0 ** -20, 1.0 + 2.0 ** -20, 4.0 + 2.0 ** -18]])
    for v in vals.astype(np.float32):
        a = abs(float(v))
        lo = max(l for l in LEVELS if l <= a)
        hi = min(l for l in LEVELS if l >= a)
        if hi == lo:
            continue
        x = (a - lo) / (hi - lo) * 65536
        n = _up_count(float(v))
        assert x - 1 < n <= x, (v, n, x)
    assert _up_count(9.0) == 0 and abs(_val(O.e2m1_sr(np.float32([9.0]), [0]))[0]) == 6.0


def test_extreme_draws():
    """The draw 0 rounds every interior value down; the draw 2^16 - 1 rounds
    up exactly the values at least 2^-16 of the gap above the lower level."""
    rng = np.random.default_rng(7)
    v = np.concatenate([rng.uniform(-6.0, 6.0, 4096),
                        2.0 ** -np.arange(2, 150, dtype=np.float64),
                        -(2.0 ** -np.arange(2, 150, dtype=np.float64)),
                        rng.uniform(0.0, 1e-30, 256)]).astype(np.float32)
    lv = np.array(LEVELS)
    keep = (np.abs(v) > 0) & (np.abs(v) < 6.0) & ~np.isin(np.abs(v).astype(np.float64), lv)
    v = v[keep]
    a = np.abs(v).astype(np.float64)
    hi = np.array([lv[lv > x].min() for x in a])
    lo = np.array([lv[lv < x].max() for x in a])
    down = np.abs(_val(O.e2m1_sr(v, np.zeros(v.size, np.uint16))))
    top = np.abs(_val(O.e2m1_sr(v, np.full(v.size, 65535, np.uint16))))
    assert np.array_equal(down, lo)
    want = np.where((a - lo) / (hi - lo) >= 2.0 ** -16, hi, lo)
    assert np.array_equal(top, want)


def test_monotone_in_v_for_fixed_draw():
    rng = np.random.default_rng(4)
    v = np.sort(rng.uniform(-7, 7, 5000).astype(np.float32))
    for _ in range(8):
        u = np.full(v.size, rng.integers(0, 2**16), np.uint16)
        out = _val(O.e2m1_sr(v, u))
        assert np.all(np.diff(out) >= 0)


def test_unbiased_over_4096_seeds():
    vals = np.array([0.1, 0.37, 0.8, 1.1, 1.3, 1.9, 2.2, 2.75, 3.3, 3.9, 4.5, 5.9,
                     -0.6, -2.6, -4.1], np.float32)
    nseed = 4096
    for k, v in enumerate(vals):
        u = np.array([O.draws16(seed, 7, k, 1)[0] for seed in range(nseed)], np.uint16)
        out = _val(O.e2m1_sr(np.full(nseed, v, np.float32), u))
        a = abs(float(v))
        lo = max(l for l in LEVELS if l <= a)
        hi = min(l for l in LEVELS if l >= a)
        p = (a - lo) / (hi - lo)
        sigma = (hi - lo) * np.sqrt(p * (1 - p) / nseed)
        assert abs(out.mean() - float(v)) <= 3 * sigma, (v, out.mean(), sigma)


def test_16_bit_draws_are_halves_of_the_32_bit_draws():
    """Draw i of the 16-bit stochastic-rounding stream is the low (i even) or
    high (i odd) half of the 32-bit draw i / 2, which the known answers
    below pin to an independent Philox4x32-10: one Philox block gives the
    draws of eight consecutive elements."""
    for seed, stream, i0 in ((0, 0, 0), (0x0123456789ABCDEF, 3, 8 * 12345), (2**64 - 1, 2, 2**35)):
        d32 = O.draws(seed, stream, i0 // 2, 64)
        d16 = O.draws16(seed, stream, i0, 128)
        want = np.stack([d32 & 0xFFFF, d32 >> 16], axis=1).reshape(-1)
        assert np.array_equal(d16.astype(np.uint32), want)


def test_philox_structure_and_determinism():
    seed, stream = 0x1234_5678_9ABC_DEF0, 11
    d = O.draws(seed, stream, 0, 64)
    for i in range(64):
        c = i // 4
        w = O.philox4x32_10([c & 0xFFFFFFFF, c >> 32, stream, 0],
                            [seed & 0xFFFFFFFF, seed >> 32])
        assert d[i] == w[i % 4]
    assert np.array_equal(d, O.draws(seed, stream, 0, 64))
    # counter high word is used: index 2^34 differs from index 0
    assert O.draws(seed, stream, 1 << 34, 4).tolist() != d[:4].tolist()
    # different streams / seeds give different sequences
    assert not np.array_equal(d, O.draws(seed, stream + 1, 0, 64))
    assert not np.array_equal(d, O.draws(seed + 1, stream, 0, 64))
    assert not np.array_equal(d, O.draws(seed ^ (1 << 40), stream, 0, 64))


def test_philox_uniformity_and_bit_balance():
    n = 1 << 20
    d = O.draws(7, 3, 0, n)
    # chi-square over 256 equal bins of the top byte
    counts = np.bincount((d >> 24).astype(np.int64), minlength=256)
    exp = n / 256
    chi2 = ((counts - exp) ** 2 / exp).sum()
    assert 150 < chi2 < 380          # dof 255: mean 255, sd ~22.6
    # every bit position is balanced (|z| < 5)
    for b in range(32):
        ones = int(((d >> b) & 1).sum())
        z = (ones - n / 2) / np.sqrt(n / 4)
        assert abs(z) < 5, (b, z)
    # consecutive draws are uncorrelated
    x = d.astype(np.float64) / 2**32 - 0.5
    r = np.corrcoef(x[:-1], x[1:])[0, 1]
    assert abs(r) < 5 / np.sqrt(n)


# --- known answers from an independent Philox4x32-10: cuRAND's host generator
def _curand():
    """cuRAND (CUDA toolkit or the nvidia-curand wheel), or None."""
    import ctypes
    import glob
    import os
    cands = []
    for root in (os.environ.get("CUDA_HOME", ""), "/usr/local/cuda"):
        if root:
            cands += sorted(glob.glob(os.path.join(root, "lib64", "libcurand.so*")))
    try:
        import nvidia.curand
        cands += sorted(glob.glob(os.path.join(nvidia.curand.__path__[0], "lib", "libcurand.so*")))
    except ImportError:
        pass
    for c in cands:
        try:
            return ctypes.CDLL(c)
        except OSError:
            continue
    return None


def _curand_philox_blocks(seed: int, n_blocks: int):
    """n_blocks 4-word outputs of cuRAND's host CURAND_RNG_PSEUDO_PHILOX4_32_10
    generator for `seed` (runs on the CPU; no GPU needed)."""
    import ctypes as C
    import pytest
    cr = _curand()
    if cr is None:
        pytest.skip("libcurand not found")
    gen = C.c_void_p()
    if cr.curandCreateGeneratorHost(C.byref(gen), 161) != 0:   # PHILOX4_32_10
        pytest.skip("cuRAND host generator unavailable")
    try:
        assert cr.curandSetPseudoRandomGeneratorSeed(gen, C.c_ulonglong(seed)) == 0
        buf = np.empty(4 * n_blocks, np.uint32)
        assert cr.curandGenerate(gen, buf.ctypes.data_as(C.c_void_p), C.c_size_t(buf.size)) == 0
    finally:
        cr.curandDestroyGenerator(gen)
    return buf.reshape(-1, 4)


def test_philox_matches_curand_host_generator():
    """cuRAND's Philox4x32-10 keys the generator with the 64-bit seed (low
    word first) and lays its output out as S parallel subsequences: output
    block c * S + s is the Philox block of counter (c, 0, s, 0).  The oracle's
    draw i of stream s is word i mod 4 of counter (i / 4, 0, s, 0), so both
    must agree block for block wherever the layouts meet.  A wrong round
    count, multiplier, Weyl constant, word order or key schedule in the
    oracle breaks the agreement everywhere."""
    for seed in (0, 0x0123456789ABCDEF, 2**64 - 1):
        blocks = _curand_philox_blocks(seed, 3 * 65536)
        key = [seed & 0xFFFFFFFF, seed >> 32]
        # the very first block is counter 0 of subsequence 0
        assert np.array_equal(blocks[0], O.philox4x32_10([0, 0, 0, 0], key))
        # the layout's width S: where counter 1 of subsequence 0 sits
        hit = np.where((blocks == O.philox4x32_10([1, 0, 0, 0], key)).all(axis=1))[0]
        assert hit.size == 1
        S = int(hit[0])
        assert S > 0 and blocks.shape[0] >= 2 * S
        rng = np.random.default_rng(seed & 0xFFFF)
        for s in list(rng.integers(0, S, 24)) + [0, 1, 2, 3, S - 1]:
            for c in (0, 1):
                want = blocks[c * S + int(s)]
                assert np.array_equal(O.philox4x32_10([c, 0, int(s), 0], key), want), (seed, c, s)
                # the oracle's draws of stream s, elements 4c .. 4c + 3
                assert np.array_equal(O.draws(seed, int(s), 4 * c, 4), want), (seed, c, s)
