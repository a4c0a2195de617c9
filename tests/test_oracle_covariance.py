"""Pins of the oracle's covariance step.

KronQ summary (hyper.ai), "Method", Eq. 7: the empirical Fisher
E[vec(g x^T) vec(g x^T)^T] factorises into H_X (x) H_G when x and g are
independent.  Checked by brute force: over the full set of (x_a, g_b) pairs
the factorisation is exact; over paired independent draws it holds to
sampling error.
"""

import numpy as np
import pytest

from oracle import covariance as cov


def _rng(s):
    return np.random.default_rng(s)


def test_kfac_exact_on_full_pair_set():
    r = _rng(1)
    xs = r.standard_normal((5, 3))    # n = 3 inputs
    gs = r.standard_normal((4, 2))    # m = 2 outputs
    pairs_x = [x for x in xs for _ in gs]
    pairs_g = [g for _ in xs for g in gs]
    F = cov.empirical_fisher(pairs_x, pairs_g)
    K = cov.kfac(cov.covariance(xs), cov.covariance(gs))
    assert F.shape == (6, 6)
    np.testing.assert_allclose(F, K, rtol=0, atol=1e-13)


def test_kfac_vec_order_matters():
    # the row-stacking vec gives H_G (x) H_X instead; with distinct factors they differ
    r = _rng(2)
    xs = r.standard_normal((6, 3)) * np.array([1.0, 3.0, 0.2])
    gs = r.standard_normal((5, 2)) * np.array([5.0, 0.1])
    pairs_x = [x for x in xs for _ in gs]
    pairs_g = [g for _ in xs for g in gs]
    F = cov.empirical_fisher(pairs_x, pairs_g)
    wrong = np.kron(cov.covariance(gs), cov.covariance(xs))
    assert np.abs(F - wrong).max() > 1e-2


def test_kfac_sampling_error_on_independent_pairs():
    r = _rng(3)
    N = 40000
    xs = r.standard_normal((N, 3)) * np.array([1.0, 2.0, 0.5])
    gs = r.standard_normal((N, 2)) * np.array([0.3, 1.5])
    F = cov.empirical_fisher(xs[:4000], gs[:4000])
    K = cov.kfac(cov.covariance(xs[:4000]), cov.covariance(gs[:4000]))
    # independent x and g: agreement to O(1/sqrt(N)) relative to the scale
    assert np.abs(F - K).max() / np.abs(K).max() < 0.1


def test_covariance_matches_loop_sum():
    r = _rng(4)
    A = r.standard_normal((37, 5))
    ref = np.zeros((5, 5))
    for t in range(A.shape[0]):
        for i in range(5):
            for j in range(5):
                ref[i, j] += A[t, i] * A[t, j]
    ref /= A.shape[0]
    np.testing.assert_allclose(cov.covariance(A), ref, rtol=1e-14, atol=1e-14)


def test_covariance_symmetric_psd_and_stream():
    r = _rng(5)
    A = r.standard_normal((300, 20)) * r.uniform(0.1, 10, 20)
    H = cov.covariance(A)
    assert np.array_equal(H, H.T) or np.abs(H - H.T).max() < 1e-12
    assert np.linalg.eigvalsh(H).min() > -1e-10
    Hs = cov.covariance_stream([A[:100], A[100:250], A[250:]], 20, 300)
    np.testing.assert_allclose(Hs, H, rtol=1e-12, atol=1e-12)
    rows = np.array([1, 5, 7])
    cols = np.array([0, 19])
    B = cov.covariance_block([A[:150], A[150:]], rows, cols, 300)
    np.testing.assert_allclose(B, H[np.ix_(rows, cols)], rtol=1e-12, atol=1e-12)


def test_covariance_empty():
    H = cov.covariance(np.zeros((0, 4)))
    assert H.shape == (4, 4) and not H.any()


@pytest.mark.parametrize("bad", [0])
def test_vec_is_column_stacking(bad):
    M = np.array([[1, 2, 3], [4, 5, 6]])
    assert list(cov.vec(M)) == [1, 4, 2, 5, 3, 6]
    g, x = np.array([1.0, 2.0]), np.array([3.0, 4.0, 5.0])
    np.testing.assert_array_equal(cov.vec(np.outer(g, x)), np.kron(x, g))


def test_streamed_diagonal_matches_the_covariance():
    r = np.random.default_rng(4)
    A = r.standard_normal((301, 37))
    chunks = [A[:100], A[100:101], A[101:]]
    np.testing.assert_allclose(cov.covariance_diag(chunks, 37, 301), np.diag(cov.covariance(A)),
                               rtol=1e-13)
