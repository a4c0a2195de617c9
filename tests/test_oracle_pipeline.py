"""Pins of the oracle's composed chain (oracle/pipeline.py, the GPTAQ chain
in oracle/gptaq.py, the deploy weights in oracle/deploy.py), each against a
property that holds whatever the composition's code looks like:

* the streamed covariance (token chunks summed, then 1/N) equals the
  covariance of the whole input, and its trace is the mean squared row norm;
* Theorem 1 of the KronQ review (pith.science), appendix: BiIP preserves the
  layer loss, so the chain's loss in the rotated space equals
  tr(H_G dW H_X dW^T) in the original space once the quantized weights are
  mapped back with the inverse transforms;
* Proposition 1 of the KronQ summary (hyper.ai), "Method": rows of W' are
  quantized independently, so any row subset reproduces those rows;
* without input drift (X~ = X) the GPTAQ chain's correction P is zero and the
  chain gives the plain chain's codes;
* the packed codes, dequantized and mapped back, are the solver's own
  reconstruction mapped back."""

import dataclasses

import numpy as np
import pytest

import synth
from oracle import biip as obiip
from oracle import deploy as odeploy
from oracle import gptaq as ogptaq
from oracle import pack as opack
from oracle import pipeline as opipe
from oracle import quantizer as oq


@pytest.fixture(scope="module")
def toy():
    cfg = synth.get_config("toy-256")
    sub = cfg.sublayers[0]
    site = cfg.site(sub.site)
    HX = opipe.x_covariance(cfg, site)
    HG = opipe.g_covariance(cfg, sub)
    return cfg, sub, site, HX, HG


def test_streamed_covariance_equals_the_whole_input():
    """Three chunks, the last one ragged: the sum over chunks divided by the
    total count (not per chunk) is X^T X / N of the whole matrix."""
    cfg = dataclasses.replace(synth.get_config("toy-256"), tokens=2 * synth.CHUNK_TOKENS + 37)
    site, sub = cfg.sites[0], cfg.sublayers[0]
    X = synth.bf16_bits_to_f32(synth.make_x(cfg, site)).astype(np.float64)
    G = synth.bf16_bits_to_f32(synth.make_g(cfg, sub)).astype(np.float64)
    N = cfg.tokens
    HX = opipe.x_covariance(cfg, site, threads=3)
    HG = opipe.g_covariance(cfg, sub, threads=2)
    np.testing.assert_allclose(HX, X.T @ X / N, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(HG, G.T @ G / N, rtol=1e-12, atol=1e-20)
    # trace = mean squared row norm; symmetric
    assert np.trace(HX) == pytest.approx(np.sum(X * X) / N, rel=1e-12)
    np.testing.assert_array_equal(HX, HX.T)


def test_chain_loss_is_the_original_space_loss(toy):
    cfg, sub, site, HX, HG = toy
    out = opipe.quantize_sublayer(cfg, sub, HX, HG, sub.bits)
    W = synth.make_w(cfg, sub).astype(np.float64)
    su, sv = synth.make_signs(cfg, sub)
    W_hat = obiip.unbiip_w(out["W_hat"], out["S_X"], out["S_G"], su, sv, cfg.mode)
    dW = W - W_hat
    loss = float(np.trace(HG @ dW @ HX @ dW.T))
    assert loss > 0
    assert out["loss"] == pytest.approx(loss, rel=1e-9)


def test_chain_row_subset_reproduces_those_rows(toy):
    cfg, sub, site, HX, HG = toy
    full = opipe.quantize_sublayer(cfg, sub, HX, HG, sub.bits)
    rows = np.array([0, 3, 100, 254, 255])
    part = opipe.quantize_sublayer(cfg, sub, HX, HG, sub.bits, rows=rows)
    np.testing.assert_array_equal(part["codes"], full["codes"][rows])
    np.testing.assert_array_equal(part["W_hat"], full["W_hat"][rows])
    # the plain-C loop gives the same rows bit for bit
    c = opipe.quantize_sublayer(cfg, sub, HX, HG, sub.bits, rows=rows, loop="c")
    np.testing.assert_array_equal(c["codes"], full["codes"][rows])


def test_gptaq_chain_without_drift_is_the_plain_chain(toy):
    cfg, sub, site, HX, HG = toy
    X_bits = synth.make_x(cfg, site)
    G_bits = synth.make_g(cfg, sub)
    res = ogptaq.chain(cfg, sub, X_bits, X_bits, G_bits, sub.bits)
    assert not np.any(res["A"]) and not np.any(res["P"])
    plain = opipe.quantize_sublayer(cfg, sub, res["HX"], res["HG"], sub.bits)
    np.testing.assert_array_equal(res["codes"], plain["codes"])
    assert res["loss"] == pytest.approx(plain["loss"], rel=1e-12)


def test_gptaq_row_subset_matches_the_full_loop():
    r = np.random.default_rng(5)
    m, n = 40, 24
    W = r.standard_normal((m, n))
    A = r.standard_normal((n, n)) * 0.05
    B = r.standard_normal((n, n))
    H = B @ B.T / n + np.eye(n)
    from oracle import cholesky as ochol
    U = ochol.inverse_cholesky(H)
    P = ogptaq.correction(A, U, 0.25)
    full = ogptaq.obs_quantize_gptaq(W, U, P, 3, group=8)
    rows = np.array([1, 7, 8, 39])
    part = ogptaq.obs_quantize_gptaq_rows(W, U, P, 3, group=8, rows=rows, chunk=3, threads=2)
    for k in ("codes", "scale", "zero", "W_hat"):
        np.testing.assert_array_equal(part[k], full[k][rows])


def test_deploy_weights_are_the_solver_reconstruction(toy):
    cfg, sub, site, HX, HG = toy
    out = opipe.quantize_sublayer(cfg, sub, HX, HG, sub.bits)
    su, sv = synth.make_signs(cfg, sub)
    Wd = odeploy.deploy_weights(opack.pack(out["codes"], sub.bits), sub.n, sub.bits, sub.group,
                                out["scale"], out["zero"], out["S_X"], out["S_G"], su, sv, cfg.mode)
    ref = obiip.unbiip_w(out["W_hat"], out["S_X"], out["S_G"], su, sv, cfg.mode)
    np.testing.assert_allclose(Wd, ref, rtol=0, atol=1e-6 * np.abs(ref).max())


def test_clip_ratios_hand_worked():
    """p_i = 1 - i/100 rounded to fp32: the first, a middle and the last of
    the 80 candidates."""
    assert oq.clip_ratio(0) == np.float32(1.0)
    assert oq.clip_ratio(6) == np.float32(0.94)
    assert oq.clip_ratio(79) == np.float32(0.21)
    assert all(oq.clip_ratio(i) > oq.clip_ratio(i + 1) for i in range(79))
