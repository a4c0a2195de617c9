"""Pins of the GPTAQ asymmetric correction in the oracle (oracle/gptaq.py).

KronQ review (pith.science), appendix, Algorithm 2, step 3:
P = alpha (Delta X X^T L) (.) M_U L^T; KronQ summary (hyper.ai), "Method":
the asymmetric-calibration objective and the compensation after quantizing
column p with delta_p and P.  What fixes each part:
  * no drift (X~ = X): P = 0 and the loop is the plain column loop, bit for bit;
  * each row p of P / alpha equals a brute-force damped least-squares fit of
    input channel p's drift onto the drifted channels p, p+1, ... over the
    explicit tokens (no Cholesky factor involved), and P is upper triangular;
  * the sign and orientation of the correction: over seeded toy layers the
    corrected loop lowers the asymmetric objective ||W_hat X~ - W X||^2 that
    the uncorrected loop leaves (a flipped sign or a transposed P raises it);
  * the BiIP of Delta X X^T is the rotation of H_X's input side: it equals
    the drift covariance of the rotated, rescaled inputs;
  * exhaustive search over all codes of tiny layers bounds the loop's loss.
"""

import itertools

import numpy as np
import pytest

import synth
from oracle import biip as obiip
from oracle import cholesky as ochol
from oracle import gptaq as G
from oracle import quantizer as Q


def _layer(r, n, N, m=6, drift=0.1):
    Xq = r.standard_normal((N, n)) * np.exp(r.uniform(-1, 1, n))[None, :]
    X = Xq + drift * r.standard_normal((N, n))
    W = r.standard_normal((m, n))
    return W, X, Xq


def test_no_drift_is_the_plain_loop():
    r = np.random.default_rng(0)
    W, _, Xq = _layer(r, 32, 200, m=9)
    H = ochol.damp(Xq.T @ Xq / len(Xq), 0.01)
    U = ochol.inverse_cholesky(H)
    P = G.correction(G.drift_covariance(Xq, Xq), U, 0.25)
    assert np.all(P == 0.0)
    for bits, group in ((4, -1), (2, 16)):
        a = G.obs_quantize_gptaq(W, U, P, bits, group)
        b = Q.obs_quantize(W, U, bits, group)
        for k in ("codes", "scale", "zero", "W_hat"):
            assert np.array_equal(a[k], b[k]), k


@pytest.mark.parametrize("n,N,lam", [(5, 40, 0.01), (12, 300, 0.01), (9, 8, 0.1)])
def test_rows_of_p_are_damped_least_squares_fits(n, N, lam):
    r = np.random.default_rng(n + N)
    _, X, Xq = _layer(r, n, N)
    H = Xq.T @ Xq / N
    delta = lam * float(np.mean(np.diag(H)))
    U = ochol.inverse_cholesky(H + delta * np.eye(n))
    alpha = 0.7
    P = G.correction(G.drift_covariance(X, Xq), U, alpha)
    assert np.allclose(np.tril(P, -1), 0.0, atol=1e-14)
    D = X - Xq
    for p in range(n):
        # min_c (1/N) ||D[:, p] - Xq[:, p:] c||^2 + delta ||c||^2, as one
        # stacked least-squares problem over the explicit tokens
        Aaug = np.vstack([Xq[:, p:] / np.sqrt(N), np.sqrt(delta) * np.eye(n - p)])
        baug = np.concatenate([D[:, p] / np.sqrt(N), np.zeros(n - p)])
        c = np.linalg.lstsq(Aaug, baug, rcond=None)[0]
        np.testing.assert_allclose(P[p, p:], alpha * c, rtol=1e-9, atol=1e-12)


def test_correction_lowers_the_asymmetric_objective():
    r = np.random.default_rng(5)
    gain = []
    for _ in range(40):
        n, N = 24, 600
        W, X, Xq = _layer(r, n, N, m=8, drift=0.3)
        H = ochol.damp(Xq.T @ Xq / N, 0.01)
        U = ochol.inverse_cholesky(H)
        A = G.drift_covariance(X, Xq)
        base = G.asymmetric_loss(Q.obs_quantize(W, U, 3)["W_hat"], W, X, Xq)
        corr = G.asymmetric_loss(G.obs_quantize_gptaq(W, U, G.correction(A, U, 1.0), 3)["W_hat"],
                                 W, X, Xq)
        flip = G.asymmetric_loss(
            G.obs_quantize_gptaq(W, U, -G.correction(A, U, 1.0), 3)["W_hat"], W, X, Xq)
        transposed = G.asymmetric_loss(
            G.obs_quantize_gptaq(W, U, G.correction(A.T, U, 1.0), 3)["W_hat"], W, X, Xq)
        gain.append((base, corr, flip, transposed))
    g = np.array(gain)
    assert g[:, 1].sum() < g[:, 0].sum()          # the correction helps on the whole
    assert g[:, 1].sum() < g[:, 2].sum()          # ... and a flipped sign does worse
    assert g[:, 1].sum() < g[:, 3].sum()          # ... and so does a transposed drift term
    assert (g[:, 1] < g[:, 0]).mean() >= 0.75


def test_biip_of_drift_covariance_is_the_drift_covariance_of_rotated_inputs():
    r = np.random.default_rng(8)
    n, N = 16, 120
    W, X, Xq = _layer(r, n, N, m=8)
    sv = (1 - 2 * r.integers(0, 2, n)).astype(np.int8)
    su = (1 - 2 * r.integers(0, 2, 8)).astype(np.int8)
    HX = Xq.T @ Xq / N
    HG = np.eye(8)
    _, HXr, _, SX, _ = obiip.biip(W, HX, HG, su, sv, 0.25, "full")
    from oracle import transform
    # the rotated, rescaled token vectors x' = V S_X^-1 x
    Xr = transform.apply(X / SX[None, :], sv)
    Xqr = transform.apply(Xq / SX[None, :], sv)
    np.testing.assert_allclose(G.rotate_like_hx(G.drift_covariance(X, Xq), SX, sv),
                               G.drift_covariance(Xr, Xqr), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(HXr, Xqr.T @ Xqr / N, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_exhaustive_search_bounds_the_corrected_loop(seed):
    r = np.random.default_rng(40 + seed)
    n, N, bits = 4, 60, 2
    W, X, Xq = _layer(r, n, N, m=1, drift=0.3)
    H = ochol.damp(Xq.T @ Xq / N, 0.01)
    U = ochol.inverse_cholesky(H)
    res = G.obs_quantize_gptaq(W, U, G.correction(G.drift_covariance(X, Xq), U, 1.0), bits)
    scale, zero = res["scale"][0, 0], int(res["zero"][0, 0])
    best = min(G.asymmetric_loss(scale * (np.array(c)[None, :] - zero), W, X, Xq)
               for c in itertools.product(range(2 ** bits), repeat=n))
    assert best <= G.asymmetric_loss(res["W_hat"], W, X, Xq) + 1e-12


def test_drifted_inputs_are_seeded_and_small():
    cfg = synth.get_config("toy-256")
    site = cfg.sites[0]
    a = synth.xq_chunk(cfg, site, 0)
    b = synth.xq_chunk(cfg, site, 0)
    assert np.array_equal(a, b)
    x = synth.bf16_bits_to_f32(synth.x_chunk(cfg, site, 0))
    xq = synth.bf16_bits_to_f32(a)
    d = xq - x
    normal = np.setdiff1d(np.arange(site.width), synth.gen.outlier_channels(cfg, site))
    assert abs(d[:, normal].std() - synth.gen.DRIFT_SIGMA) < 0.01
