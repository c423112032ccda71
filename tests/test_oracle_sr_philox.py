"""Pins for the oracle's stochastic rounding and its Philox4x32-10 draws.

Stochastic rounding ("FP4 All the Way", Key points: stochastic rounding for
the backward and update passes) is pinned by what the definition of an
unbiased stochastic rounding fixes: lattice points are fixed, the rounding
is unbiased (mean over 4096 seeds within 3 sigma), the up-probability is the
exact fraction of the gap, and for a fixed draw the result is monotone in v.
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
    u = np.random.default_rng(0).integers(0, 2**32, 64, dtype=np.uint64).astype(np.uint32)
    for lv in LEVELS:
        for s in (1.0, -1.0):
            v = np.full(64, s * lv, np.float32)
            out = _val(O.e2m1_sr(v, u))
            assert np.all(out == s * lv)


def test_up_probability_is_exact_fraction_of_gap():
    # v = 1.25 sits at p = 1/2 of the gap [1, 1.5]: up iff u < 2^31
    v = np.full(4, 1.25, np.float32)
    u = np.array([0, 2**31 - 1, 2**31, 2**32 - 1], np.uint32)
    assert list(_val(O.e2m1_sr(v, u))) == [1.5, 1.5, 1.0, 1.0]
    # v = 2.25 is p = 1/4 of [2, 3]: up iff u < 2^30
    v = np.full(3, 2.25, np.float32)
    u = np.array([2**30 - 1, 2**30, 0], np.uint32)
    assert list(_val(O.e2m1_sr(v, u))) == [3.0, 2.0, 3.0]
    # v = 5.5 is p = 3/4 of [4, 6]: up iff u < 3 * 2^30
    v = np.full(2, 5.5, np.float32)
    u = np.array([3 * 2**30 - 1, 3 * 2**30], np.uint32)
    assert list(_val(O.e2m1_sr(v, u))) == [6.0, 4.0]
    # beyond 6 saturates; a tiny positive value rounds up only for u = 0
    assert list(_val(O.e2m1_sr(np.array([9.0, 1e-30, 1e-30], np.float32),
                               np.array([0, 0, 1], np.uint32)))) == [6.0, 0.5, 0.0]


def test_extreme_draws_decide_every_interior_value():
    """Strictly between two levels 0 < p < 1, so ceil(p * 2^32) lies in
    [1, 2^32 - 1]: the draw 0 always rounds up and the draw 2^32 - 1 never
    does, down to p of a single binary32 subnormal (a rounded-down threshold
    would send the smallest p to the lower level with every draw)."""
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
    up = np.abs(_val(O.e2m1_sr(v, np.zeros(v.size, np.uint32))))
    down = np.abs(_val(O.e2m1_sr(v, np.full(v.size, 2**32 - 1, np.uint32))))
    assert np.array_equal(up, hi)
    assert np.array_equal(down, lo)


def test_monotone_in_v_for_fixed_draw():
    rng = np.random.default_rng(4)
    v = np.sort(rng.uniform(-7, 7, 5000).astype(np.float32))
    for _ in range(8):
        u = np.full(v.size, rng.integers(0, 2**32, dtype=np.uint64), np.uint32)
        out = _val(O.e2m1_sr(v, u))
        assert np.all(np.diff(out) >= 0)


def test_unbiased_over_4096_seeds():
    vals = np.array([0.1, 0.37, 0.8, 1.1, 1.3, 1.9, 2.2, 2.75, 3.3, 3.9, 4.5, 5.9,
                     -0.6, -2.6, -4.1], np.float32)
    nseed = 4096
    for k, v in enumerate(vals):
        u = np.array([O.draws(seed, 7, k, 1)[0] for seed in range(nseed)], np.uint32)
        out = _val(O.e2m1_sr(np.full(nseed, v, np.float32), u))
        a = abs(float(v))
        lo = max(l for l in LEVELS if l <= a)
        hi = min(l for l in LEVELS if l >= a)
        p = (a - lo) / (hi - lo)
        sigma = (hi - lo) * np.sqrt(p * (1 - p) / nseed)
        assert abs(out.mean() - float(v)) <= 3 * sigma, (v, out.mean(), sigma)


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
