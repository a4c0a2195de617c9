"""Pins of the oracle's randomized Hadamard transforms (textbook matrices,
orthogonality, dense vs fast)."""

import numpy as np
import pytest

from conftest import GOLDEN
from oracle import transform as T


def _load(name):
    return np.loadtxt(GOLDEN / name, comments="#")


def test_sylvester_h4_golden():
    np.testing.assert_array_equal(T.sylvester(2), _load("hadamard_4.txt"))


@pytest.mark.parametrize("k", [0, 1, 3, 6])
def test_sylvester_orthogonal(k):
    H = T.sylvester(k)
    np.testing.assert_array_equal(H @ H.T, (2 ** k) * np.eye(2 ** k))
    assert set(np.unique(H)) <= {-1.0, 1.0}


@pytest.mark.parametrize("k", [1, 4, 8])
def test_fwht_matches_dense(k):
    r = np.random.default_rng(k)
    x = r.standard_normal((3, 2 ** k))
    np.testing.assert_allclose(T.fwht(x), x @ T.sylvester(k).T, rtol=1e-12, atol=1e-12)


def test_fwht_of_unit_vector_is_flat():
    e0 = np.zeros(64)
    e0[0] = 1.0
    np.testing.assert_array_equal(T.fwht(e0), np.ones(64))
    # and a flat vector goes to a spike
    np.testing.assert_array_equal(T.fwht(np.ones(64)), 64 * e0)


def test_dct2_golden_and_orthonormal():
    np.testing.assert_allclose(T.dct2(3), _load("dct2_3.txt"), rtol=0, atol=1e-15)
    for q in (1, 2, 7, 43):
        C = T.dct2(q)
        np.testing.assert_allclose(C @ C.T, np.eye(q), atol=1e-13)
    np.testing.assert_allclose(T.dct2(2), T.sylvester(1) / np.sqrt(2), atol=1e-15)


@pytest.mark.parametrize("d", [1, 2, 3, 7, 12, 14, 43, 86, 172, 256, 448])
def test_transform_orthonormal_and_fast(d):
    r = np.random.default_rng(d)
    s = (1 - 2 * r.integers(0, 2, d)).astype(np.int8)
    M = T.dense(d, s)
    np.testing.assert_allclose(M @ M.T, np.eye(d), atol=1e-12)
    x = r.standard_normal((4, d))
    np.testing.assert_allclose(T.apply(x, s), x @ M.T, atol=1e-12)
    np.testing.assert_allclose(T.apply_t(T.apply(x, s), s), x, atol=1e-12)


def test_split_width():
    assert T.split_width(11008) == (43, 8)
    assert T.split_width(14336) == (7, 11)
    assert T.split_width(28672) == (7, 12)
    assert T.split_width(4096) == (1, 12)
    with pytest.raises(ValueError):
        T.split_width(0)


def test_power_of_two_is_normalized_hadamard():
    d = 16
    s = np.ones(d, dtype=np.int8)
    np.testing.assert_allclose(T.dense(d, s), T.sylvester(4) / 4.0, atol=1e-15)


@pytest.mark.parametrize("d", [8, 56, 344, 112])
def test_selected_rows_match_the_dense_matrix(d):
    r = np.random.default_rng(d)
    s = np.where(r.random(d) < 0.5, -1.0, 1.0)
    idx = r.choice(d, min(d, 9), replace=False)
    np.testing.assert_allclose(T.rows(d, idx, s), T.dense(d, s)[idx], atol=1e-13)
