"""Pins of the oracle's BiIP step.

KronQ review (pith.science), appendix A.2, Theorem 1: with W' = U W V^T,
H_G' = U H_G U^T, H_X' = V H_X V^T the loss tr(H_G dW H_X dW^T) is
unchanged; the diagonal rescale is loss-preserving by construction; at
alpha = 1/4 the rescale equalises the diagonal of H with the squared norms.
"""

import numpy as np
import pytest

from oracle import biip, transform
from oracle.quantizer import layer_loss


def _spd(r, d, spread=3.0):
    A = r.standard_normal((d, 3 * d)) * np.exp(r.uniform(-spread, spread, d))[:, None]
    return A @ A.T / (3 * d)


def _signs(r, d):
    return (1 - 2 * r.integers(0, 2, d)).astype(np.int8)


@pytest.mark.parametrize("m,n", [(8, 16), (7, 12), (14, 43)])
@pytest.mark.parametrize("mode", biip.MODES)
def test_theorem1_loss_invariance(m, n, mode):
    r = np.random.default_rng(m * 100 + n)
    W = r.standard_normal((m, n))
    W_hat = W + 0.05 * r.standard_normal((m, n))
    HX, HG = _spd(r, n), _spd(r, m)
    su, sv = _signs(r, m), _signs(r, n)
    Wp, HXp, HGp, SX, SG = biip.biip(W, HX, HG, su, sv, 0.25, mode)
    # the same transform applied to W_hat (linear map: rescale + rotate)
    in_s, out_s, in_r, out_r = biip.sides(mode)
    Wh = W_hat * SX[None, :] * SG[:, None]
    if in_r:
        Wh = Wh @ transform.dense(n, sv).T
    if out_r:
        Wh = transform.dense(m, su) @ Wh
    l0 = layer_loss(W - W_hat, HX, HG)
    l1 = layer_loss(Wp - Wh, HXp, HGp)
    assert abs(l1 - l0) <= 1e-10 * abs(l0)


@pytest.mark.parametrize("mode", biip.MODES)
def test_rotate_then_unrotate_identity(mode):
    r = np.random.default_rng(7)
    m, n = 12, 28
    W = r.standard_normal((m, n))
    HX, HG = _spd(r, n), _spd(r, m)
    su, sv = _signs(r, m), _signs(r, n)
    Wp, _, _, SX, SG = biip.biip(W, HX, HG, su, sv, 0.25, mode)
    np.testing.assert_allclose(biip.unbiip_w(Wp, SX, SG, su, sv, mode), W, atol=1e-12)


def test_dense_matches_fast_rotation():
    r = np.random.default_rng(8)
    m, n = 14, 24
    W = r.standard_normal((m, n))
    HX, HG = _spd(r, n), _spd(r, m)
    su, sv = _signs(r, m), _signs(r, n)
    Wp, HXp, HGp = biip.rotate(W, HX, HG, su, sv)
    U, V = transform.dense(m, su), transform.dense(n, sv)
    np.testing.assert_allclose(Wp, U @ W @ V.T, atol=1e-12)
    np.testing.assert_allclose(HXp, V @ HX @ V.T, atol=1e-12)
    np.testing.assert_allclose(HGp, U @ HG @ U.T, atol=1e-12)
    np.testing.assert_allclose(U @ U.T, np.eye(m), atol=1e-12)
    np.testing.assert_allclose(V @ V.T, np.eye(n), atol=1e-12)


def test_alpha_quarter_equalisation():
    r = np.random.default_rng(9)
    m, n = 16, 32
    W = r.standard_normal((m, n)) * np.exp(r.uniform(-2, 2, n))[None, :]
    HX, HG = _spd(r, n), _spd(r, m)
    # input side alone: diag(H_X') == column norms^2 of W'
    W1, HX1, _, SX, SG = biip.rescale(W, HX, HG, 0.25, "sv_only")
    np.testing.assert_allclose(np.diag(HX1), (W1 ** 2).sum(0), rtol=1e-12)
    assert np.all(SG == 1)
    # full: the output side comes last, so diag(H_G') == row norms^2 of W'
    W2, _, HG2, SX2, SG2 = biip.rescale(W, HX, HG, 0.25, "full")
    np.testing.assert_allclose(np.diag(HG2), (W2 ** 2).sum(1), rtol=1e-12)
    np.testing.assert_allclose(SX2, (np.diag(HX) / (W ** 2).sum(0)) ** 0.25, rtol=1e-14)
    # and alpha = 0 is the identity
    W0, HX0, HG0, SX0, SG0 = biip.rescale(W, HX, HG, 0.0, "full")
    assert np.all(SX0 == 1) and np.all(SG0 == 1)
    np.testing.assert_array_equal(W0, W)


def test_alpha_half_exchanges_diagonal_and_norms():
    """KronQ README (GitHub), "Mapping paper results to flags": the
    weight-and-activation setting uses --alpha 0.5.  At alpha = 1/2 the input
    rescale S_X = (H_jj / ||W_j||^2)^(1/2) exchanges the two: the rescaled
    diagonal H_jj / S_j^2 is the old squared column norm and the rescaled
    squared column norm ||W_j||^2 S_j^2 is the old diagonal (closed form)."""
    r = np.random.default_rng(19)
    m, n = 12, 24
    W = r.standard_normal((m, n)) * np.exp(r.uniform(-2, 2, n))[None, :]
    HX, HG = _spd(r, n), _spd(r, m)
    W1, HX1, _, SX, _ = biip.rescale(W, HX, HG, 0.5, "sv_only")
    np.testing.assert_allclose(np.diag(HX1), (W ** 2).sum(0), rtol=1e-12)
    np.testing.assert_allclose((W1 ** 2).sum(0), np.diag(HX), rtol=1e-12)


def test_modes_touch_only_their_side():
    r = np.random.default_rng(10)
    m, n = 8, 16
    W = r.standard_normal((m, n))
    HX, HG = _spd(r, n), _spd(r, m)
    su, sv = _signs(r, m), _signs(r, n)
    _, HXp, HGp, SX, SG = biip.biip(W, HX, HG, su, sv, 0.25, "no_rescale")
    assert np.all(SX == 1) and np.all(SG == 1)
    _, HXp, HGp, SX, SG = biip.biip(W, HX, HG, su, sv, 0.25, "sv_only")
    np.testing.assert_array_equal(HGp, HG)
    assert np.all(SG == 1)
    _, HXp, HGp, SX, SG = biip.biip(W, HX, HG, su, sv, 0.25, "su_only")
    np.testing.assert_array_equal(HXp, HX)
    assert np.all(SX == 1)
    with pytest.raises(ValueError):
        biip.sides("bogus")


def test_zero_guards():
    W = np.array([[1.0, 0.0], [2.0, 0.0]])
    HX = np.diag([4.0, 0.0])
    HG = np.diag([1.0, 1.0])
    _, _, _, SX, SG = biip.rescale(W, HX, HG, 0.25, "full")
    assert SX[1] == 1.0 and SX[0] != 1.0


def test_rotation_spreads_a_spike():
    # incoherence: a coordinate-aligned H becomes flat on the diagonal
    n = 64
    r = np.random.default_rng(11)
    HX = np.diag(np.r_[1000.0, np.ones(n - 1)])
    _, HXp, _ = biip.rotate(np.zeros((4, n)), HX, np.eye(4), _signs(r, 4), _signs(r, n))
    d = np.diag(HXp)
    np.testing.assert_allclose(d, np.full(n, np.trace(HX) / n), rtol=1e-12)


@pytest.mark.parametrize("m,n", [(56, 64), (16, 344), (86, 28)])
@pytest.mark.parametrize("mode", ["full", "no_rescale", "su_only", "sv_only"])
def test_sampled_entries_equal_the_whole_transform(m, n, mode):
    """The selected-entries form (used at widths where the whole fp64
    transform is too slow) equals rescale + rotate, including odd factors."""
    r = np.random.default_rng(m * n)
    W = r.standard_normal((m, n)) * np.exp(r.uniform(-1, 1, n))[None, :]
    HX, HG = _spd(r, n), _spd(r, m)
    su, sv = _signs(r, m), _signs(r, n)
    Wp, HXp, HGp, SX, SG = biip.biip(W, HX, HG, su, sv, 0.25, mode)
    wr, wc = r.choice(m, 7, replace=False), r.choice(n, 9, replace=False)
    hx, hg = r.choice(n, 11, replace=False), r.choice(m, 5, replace=False)
    Wb, HXb, HGb, SXs, SGs = biip.biip_entries(W, HX, HG, su, sv, 0.25, mode, wr, wc, hx, hg)
    np.testing.assert_allclose(SXs, SX, rtol=1e-14)
    np.testing.assert_allclose(SGs, SG, rtol=1e-14)
    np.testing.assert_allclose(Wb, Wp[np.ix_(wr, wc)], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(HXb, HXp[np.ix_(hx, hx)], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(HGb, HGp[np.ix_(hg, hg)], rtol=1e-10, atol=1e-12)
