"""Pins of the incoherence diagnostics, and the pages' qualitative claims
reproduced on synthetic layers.

KronQ summary (hyper.ai), "Method"; review, Figure 2: mu(H_G)/sqrt(d_out)
near 1 before incoherence processing and small after it; BiIP lowers both
CV_in and CV_out, input-side processing alone barely moves CV_out.
"""

import numpy as np

import synth
from oracle import biip, diagnostics as D, transform


def test_mu_closed_forms():
    # a diagonal matrix with distinct entries: eigenvectors are the axes
    assert D.mu_normalized(np.diag(np.arange(1.0, 33.0))) == 1.0
    # the normalised Walsh-Hadamard basis: every |entry| is 1/sqrt(d)
    d = 64
    T = transform.dense(d)
    H = T @ np.diag(np.arange(1.0, d + 1.0)) @ T.T
    np.testing.assert_allclose(D.mu_normalized(H), 1.0 / np.sqrt(d), rtol=1e-9)


def test_cv_closed_forms():
    W = np.ones((5, 7))
    assert D.cv_in(W) == 0.0 and D.cv_out(W) == 0.0
    # row norms 1 and 3: mean 2, population std 1 -> CV 0.5
    W = np.array([[1.0, 0.0], [0.0, 3.0]])
    np.testing.assert_allclose(D.cv_out(W), 0.5, rtol=1e-15)
    np.testing.assert_allclose(D.cv_in(W), 0.5, rtol=1e-15)


def _layer(m, n, tokens, seed):
    r = np.random.default_rng(seed)
    W = (r.standard_normal((m, n)) * 0.02 * np.exp(r.uniform(np.log(0.5), np.log(2.0), m))[:, None]
         * np.exp(r.uniform(np.log(0.5), np.log(2.0), n))[None, :])
    X = r.standard_normal((tokens, n))
    X[:, r.permutation(n)[:4]] *= 20.0
    G = r.standard_normal((tokens, m)) * 10.0 ** (-3.0 * r.random(m))[None, :]
    HX = X.T @ X / tokens
    HG = G.T @ G / tokens
    su = np.where(r.random(m) < 0.5, -1, 1).astype(np.int8)
    sv = np.where(r.random(n) < 0.5, -1, 1).astype(np.int8)
    return W, HX, HG, su, sv


def test_bidirectional_processing_incoheres_H_G_and_evens_both_norms():
    m = n = 512
    W, HX, HG, su, sv = _layer(m, n, 4096, 3)
    before = D.mu_normalized(HG)
    Wf, _, HGf, _, _ = biip.biip(W, HX, HG, su, sv, 0.25, "full")
    Wv, _, HGv, _, _ = biip.biip(W, HX, HG, su, sv, 0.25, "sv_only")
    after = D.mu_normalized(HGf)
    assert before > 0.9                       # per-channel scales over 3 decades: near-diagonal
    assert after < before / 4
    assert D.mu_normalized(HGv) == before     # input-side processing leaves H_G alone
    # input-side processing lowers CV_in but leaves CV_out; BiIP lowers both
    assert D.cv_in(Wv) < 0.5 * D.cv_in(W) and D.cv_in(Wf) < 0.5 * D.cv_in(W)
    assert abs(D.cv_out(Wv) - D.cv_out(W)) < 0.25 * D.cv_out(W)
    assert D.cv_out(Wf) < 0.5 * D.cv_out(Wv)
