"""Pins for the oracle's block-wise random Hadamard transform.

The transform ("FP4", How it works: random Hadamard transforms tame
outliers; "Quartet", Approach: block-wise Hadamard rotations) is pinned
against scipy's Sylvester Hadamard matrix, orthogonality H H^T = n I, norm
preservation and invariance of a product of two rotated operands.
"""
import numpy as np
import pytest
import scipy.linalg

import oracle as O


@pytest.mark.parametrize("n", [16, 32])
def test_transform_equals_scipy_hadamard(n):
    ones = np.ones(n, np.float32)
    H = np.stack([O.rht_block(np.eye(n, dtype=np.float32)[j], n, ones) for j in range(n)])
    c = O.rht_scale(n)
    assert np.array_equal(H, (scipy.linalg.hadamard(n) * np.float32(c)).astype(np.float32))
    Hn = np.rint(H.astype(np.float64) / c)
    assert np.array_equal(Hn @ Hn.T, n * np.eye(n))


@pytest.mark.parametrize("n", [16, 32])
def test_signs_and_scale(n):
    d = O.rht_signs(5, n)
    assert set(np.unique(d).tolist()) <= {-1.0, 1.0}
    draws = O.draws(5, O.RHT_STREAM, 0, n)
    assert np.array_equal(d < 0, (draws >> 31) == 1)
    assert O.rht_scale(16) == 0.25
    assert abs(O.rht_scale(32) - 1 / np.sqrt(32)) < 1e-8


@pytest.mark.parametrize("n", [16, 32])
def test_rotated_block_matches_matrix_form(n):
    rng = np.random.default_rng(6)
    d = O.rht_signs(9, n)
    x = rng.standard_normal(n).astype(np.float32)
    y = O.rht_block(x, n, d)
    ref = (x.astype(np.float64) * d) @ scipy.linalg.hadamard(n) * (1 / np.sqrt(n))
    assert np.allclose(y, ref, rtol=1e-6, atol=1e-6)
    assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-5 * np.linalg.norm(x)


@pytest.mark.parametrize("n", [16, 32])
def test_product_invariance(n):
    rng = np.random.default_rng(7)
    X = rng.standard_normal((64, 256)).astype(np.float32)
    W = rng.standard_normal((48, 256)).astype(np.float32)
    Xr = O.rht_rows(X, n, 123)
    Wr = O.rht_rows(W, n, 123)
    ref = X.astype(np.float64) @ W.T.astype(np.float64)
    got = Xr.astype(np.float64) @ Wr.T.astype(np.float64)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-6
    # a different sign vector on one side breaks the invariance
    Wbad = O.rht_rows(W, n, 124)
    bad = Xr.astype(np.float64) @ Wbad.T.astype(np.float64)
    assert np.linalg.norm(bad - ref) / np.linalg.norm(ref) > 0.1
