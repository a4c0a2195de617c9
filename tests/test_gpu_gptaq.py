"""GPTAQ asymmetric calibration on the GPU against the fp64 oracle.

KronQ review (pith.science), appendix, Algorithm 2, step 3
(P = alpha (Delta X X^T L) (.) M_U L^T) and the column loop; KronQ summary
(hyper.ai), "Method" (the asymmetric-calibration objective).  The readings
are those of oracle/gptaq.py and include/kronq.h.

Bars: H~ <= 1e-4 relative Frobenius (a covariance); the drift covariance is
a difference of two fp32 sums of size |H|, so its relative error is the
covariance's 1e-5-level error scaled by |H| / |A| (computed here from the
oracle's values); P is checked against the oracle's P of the GPU's own A' and U_c at 1e-4
(two chained fp32-accurate tensor-core products, as H and U_c are held);
>= 99.9 % identical codes and the loss within 1 %, as for the plain solver.
"""

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import synth
from gpu_helpers import bf16_dev, rel_fro, spd, t
from oracle import cholesky as ochol
from oracle import gptaq as og
from oracle import quantizer as oq
from post_quantization_02_b200 import abi
from post_quantization_02_b200 import pipeline as gpipe

pytestmark = pytest.mark.gpu


def _side_by_side(xq_bits, x_bits):
    """Rows [x~_t, x_t] (N x 2n bf16 bits): the input kronq_drift_covariance takes."""
    return np.ascontiguousarray(np.concatenate([xq_bits, x_bits], axis=1))


def _gpu_chain(cfg, sub, dev, xb, xqb, gb, bits, alpha_asym=0.25):
    n, m = sub.n, sub.m
    XqX = bf16_dev(_side_by_side(xqb, xb), dev)
    HX = torch.empty((n, n), device=dev)
    A = torch.empty((n, n), device=dev)
    ws = abi.gptaq_workspace(m, n, dev)
    abi.kronq_drift_covariance(XqX, HX, A, ws=ws)
    del XqX
    HG = torch.empty((m, m), device=dev)
    abi.kronq_covariance(bf16_dev(gb, dev), HG, 1.0 / gb.shape[0], 0.0)
    su, sv = synth.make_signs(cfg, sub)
    res = gpipe.quantize_sublayer_gptaq(t(synth.make_w(cfg, sub), dev), HX, A, HG, t(su, dev),
                                        t(sv, dev), bits, sub.group, cfg.alpha, cfg.mode, cfg.damp,
                                        cfg.block, alpha_asym, keep=True, ws=ws)
    torch.cuda.synchronize()
    return HX, A, HG, res


@pytest.mark.parametrize("mode", ["full", "no_rescale"])
def test_toy_layer_gptaq_full_chain(cuda, mode):
    cfg = dataclasses.replace(synth.get_config("toy-256"), mode=mode)
    sub, site = cfg.sublayers[0], cfg.sites[0]
    xb, xqb, gb = synth.make_x(cfg, site), synth.make_xq(cfg, site), synth.make_g(cfg, sub)
    HX, A, HG, res = _gpu_chain(cfg, sub, cuda, xb, xqb, gb, sub.bits)
    ref = og.chain(cfg, sub, xb, xqb, gb, sub.bits)
    assert res.info.item() == 0
    eps_h = rel_fro(HX.cpu().numpy(), ref["HX"])
    assert eps_h <= 1e-4
    # A is the difference of two fp32 sums of size |H|: its absolute error is
    # at most about twice theirs
    a_bar = 2 * max(eps_h, 1e-6) * np.linalg.norm(ref["HX"]) / np.linalg.norm(ref["A"])
    assert rel_fro(A.cpu().numpy(), ref["A"]) <= a_bar, (rel_fro(A.cpu().numpy(), ref["A"]), a_bar)
    assert rel_fro(res.A.cpu().numpy(), ref["A_rot"]) <= 2 * a_bar
    # P from the GPU's own A' and U_c (stage-isolated, fp32-accurate products)
    Pr = og.correction(res.A.cpu().numpy(), res.U_c.cpu().numpy(), 0.25)
    assert rel_fro(res.P.cpu().numpy(), Pr) <= 1e-4
    assert np.all(np.tril(res.P.cpu().numpy(), -1) == 0)
    codes = res.codes.cpu().numpy()
    same = (codes == ref["codes"]).mean()
    assert same >= 0.999, same
    loss = oq.layer_loss(res.W_rot.cpu().numpy() - res.W_hat.cpu().numpy(), ref["HX_rot"],
                         ref["HG_rot"])
    assert abs(loss / ref["loss"] - 1) <= 0.01, (loss, ref["loss"])


def test_zero_drift_is_the_plain_solver_bit_for_bit(cuda):
    """X~ = X: the drift covariance is exactly zero (the two blocks of the
    side-by-side covariance are the same sums), so is P, and the solver with
    the P term returns the plain solver's codes and W_hat bit for bit."""
    cfg = synth.get_config("toy-256")
    sub, site = cfg.sublayers[0], cfg.sites[0]
    xb, gb = synth.make_x(cfg, site), synth.make_g(cfg, sub)
    HX, A, HG, res = _gpu_chain(cfg, sub, cuda, xb, xb, gb, sub.bits)
    assert torch.count_nonzero(A).item() == 0
    assert torch.count_nonzero(res.P).item() == 0
    su, sv = synth.make_signs(cfg, sub)
    plain = gpipe.quantize_sublayer(t(synth.make_w(cfg, sub), cuda), HX, HG, t(su, cuda),
                                    t(sv, cuda), sub.bits, sub.group, cfg.alpha, cfg.mode, cfg.damp,
                                    cfg.block, keep=True)
    torch.cuda.synchronize()
    assert torch.equal(plain.codes, res.codes)
    assert torch.equal(plain.W_hat, res.W_hat)


@pytest.mark.parametrize("m,n,group", [(512, 1024, -1), (300, 2048, 128), (256, 384, 128)])
def test_gptaq_solver_matches_oracle(cuda, m, n, group):
    """The solver and P alone (stage-isolated) on random layers, one- and
    two-level lazy updates (n = 384 stays inside one super-block)."""
    r = np.random.default_rng(m + n)
    H = spd(r, n, spread=1.0)
    U = ochol.inverse_cholesky(ochol.damp(H, 0.01)).astype(np.float32)
    A = (0.05 * r.standard_normal((n, n)) * np.sqrt(np.outer(np.diag(H), np.diag(H)))).astype(np.float32)
    W = (r.standard_normal((m, n)) * 0.02).astype(np.float32)
    Ud, Ad = t(U, cuda), t(A, cuda)
    P = torch.empty((n, n), device=cuda)
    ws = abi.gptaq_workspace(m, n, cuda)
    info = torch.zeros(1, dtype=torch.int32, device=cuda)
    abi.kronq_gptaq_correction(Ad, Ud, 0.5, P, info, ws)
    Pr = og.correction(A.astype(np.float64), U.astype(np.float64), 0.5)
    assert rel_fro(P.cpu().numpy(), Pr) <= 1e-4      # two chained fp32-accurate products
    G = 1 if group == -1 else n // group
    codes = torch.empty((m, n), dtype=torch.uint8, device=cuda)
    scales = torch.empty((m, G), device=cuda)
    zeros = torch.empty((m, G), dtype=torch.uint8, device=cuda)
    What = torch.empty((m, n), device=cuda)
    Wd = t(W, cuda)
    abi.kronq_quantize_layer_gptaq(Wd, Ud, P, 2, group, 128, codes, scales, zeros, What, info, ws)
    torch.cuda.synchronize()
    assert info.item() == 0
    ref = og.obs_quantize_gptaq_rows(W, U, P.cpu().numpy(), 2, group)
    same = (codes.cpu().numpy() == ref["codes"]).mean()
    assert same >= 0.999, same
    lg = oq.row_losses(W - What.cpu().numpy(), H, 0.01).sum()
    lr = oq.row_losses(W - ref["W_hat"], H, 0.01).sum()
    assert abs(lg / lr - 1) <= 0.01, (lg, lr)


def test_llama2_7b_q_proj_gptaq_rows(cuda):
    """The 4096 x 4096 layer with 262144 drifted tokens: the GPU chain in the
    order a calibration run takes it; the oracle computes P from the GPU's
    rotated H~' and drift covariance, and reruns the column loop on 1024
    seeded rows (rows are independent given U_c and P)."""
    cfg = synth.get_config("llama2-7b-q_proj")
    sub, site = cfg.sublayers[0], cfg.site("attn_in")
    N, n, m = cfg.tokens, sub.n, sub.m
    XqX = torch.empty((N, 2 * n), dtype=torch.bfloat16, device=cuda)

    def pair(c):
        xb = synth.x_chunk(cfg, site, c)
        return c, _side_by_side(synth.xq_chunk(cfg, site, c, x_bits=xb), xb)

    with ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1))) as ex:
        for c, bits in ex.map(pair, range(synth.n_chunks(N))):
            r0 = c * synth.CHUNK_TOKENS
            XqX[r0:r0 + len(bits)].copy_(bf16_dev(bits, "cpu"))
    HX = torch.empty((n, n), device=cuda)
    A = torch.empty((n, n), device=cuda)
    ws = abi.gptaq_workspace(m, n, cuda)
    abi.kronq_drift_covariance(XqX, HX, A, ws=ws)
    del XqX
    G = bf16_dev(synth.make_g(cfg, sub), cuda)
    HG = torch.empty((m, m), device=cuda)
    abi.kronq_covariance(G, HG, 1.0 / N, 0.0)
    del G
    torch.cuda.empty_cache()
    su, sv = synth.make_signs(cfg, sub)
    res = gpipe.quantize_sublayer_gptaq(t(synth.make_w(cfg, sub), cuda), HX, A, HG, t(su, cuda),
                                        t(sv, cuda), sub.bits, sub.group, cfg.alpha, cfg.mode,
                                        cfg.damp, cfg.block, 0.25, keep=True, ws=ws)
    torch.cuda.synchronize()
    assert res.info.item() == 0
    U = res.U_c.cpu().numpy().astype(np.float64)
    Pr = og.correction(res.A.cpu().numpy(), U, 0.25)
    Pg = res.P.cpu().numpy()
    assert rel_fro(Pg, Pr) <= 1e-4
    rows = np.sort(np.random.default_rng(7).choice(m, 1024, replace=False))
    Wrot = res.W_rot.cpu().numpy()
    ref = og.obs_quantize_gptaq_rows(Wrot[rows], U, Pg, sub.bits, sub.group)
    codes = res.codes.cpu().numpy()[rows]
    same = (codes == ref["codes"]).mean()
    assert same >= 0.999, same
    HXr = res.H_X.cpu().numpy()
    lg = oq.row_losses(Wrot[rows] - res.W_hat.cpu().numpy()[rows], HXr, cfg.damp).sum()
    lr = oq.row_losses(Wrot[rows] - ref["W_hat"], HXr, cfg.damp).sum()
    assert abs(lg / lr - 1) <= 0.01, (lg, lr)
