"""Whole-path parity on the toy layer: the seeded 256 x 256 layer with 2048
calibration tokens (bf16 X with 4 outlier channels, G with per-channel
scales over 3 decades, W4 asymmetric per-channel, BiIP, 1 % damping),
run through the C ABI and compared step by step with the fp64 oracle run on
the same seeded inputs.  Also the mixed-precision ranking on a small block
of sublayers that share one input."""

import dataclasses

import numpy as np
import pytest
import torch

import synth
from gpu_helpers import bf16_dev, rel_fro, t
from oracle import pipeline as opipe
from oracle import sensitivity as osens
from post_quantization_02_b200 import abi, alloc
from post_quantization_02_b200 import pipeline as gpipe

pytestmark = pytest.mark.gpu


def _gpu_layer(cfg, sub, dev, bits, keep=True):
    site = cfg.site(sub.site)
    X = bf16_dev(synth.make_x(cfg, site), dev)
    G = bf16_dev(synth.make_g(cfg, sub), dev)
    HX = gpipe.covariance(X)
    HG = gpipe.covariance(G)
    W = t(synth.make_w(cfg, sub), dev)
    su, sv = synth.make_signs(cfg, sub)
    res = gpipe.quantize_sublayer(W, HX, HG, t(su, dev), t(sv, dev), bits, sub.group, cfg.alpha,
                                  cfg.mode, cfg.damp, cfg.block, keep=keep)
    return HX, HG, res


def test_toy_layer_full_chain(cuda):
    cfg = synth.get_config("toy-256")
    sub = cfg.sublayers[0]
    HXg, HGg, res = _gpu_layer(cfg, sub, cuda, sub.bits)
    HX = opipe.x_covariance(cfg, cfg.sites[0])
    HG = opipe.g_covariance(cfg, sub)
    ref = opipe.quantize_sublayer(cfg, sub, HX, HG, sub.bits)
    assert rel_fro(HXg.cpu().numpy(), HX) <= 1e-4
    assert rel_fro(HGg.cpu().numpy(), HG) <= 1e-4
    np.testing.assert_allclose(res.S_X.cpu().numpy(), ref["S_X"], rtol=1e-4)
    np.testing.assert_allclose(res.S_G.cpu().numpy(), ref["S_G"], rtol=1e-4)
    assert rel_fro(res.W_rot.cpu().numpy(), ref["W_rot"]) <= 1e-4
    assert rel_fro(res.H_X.cpu().numpy(), ref["HX_rot"]) <= 1e-4
    assert rel_fro(res.H_G.cpu().numpy(), ref["HG_rot"]) <= 1e-4
    np.testing.assert_allclose(res.sens[0].item(), ref["s"], rtol=1e-4)
    # U_c: stage-isolated (the oracle factors the GPU's own H_X') at 1e-4;
    # end to end it also carries the difference of its input H_X', which the
    # factor of the damped matrix amplifies by at most about kappa(H_d)
    # (first-order perturbation of the factorisation)
    from oracle import cholesky as ochol
    Ug, HXr = res.U_c.cpu().numpy(), res.H_X.cpu().numpy()
    assert rel_fro(Ug, ochol.inverse_cholesky(ochol.damp(HXr, cfg.damp))) <= 1e-4
    ev = np.linalg.eigvalsh(ochol.damp(ref["HX_rot"], cfg.damp))
    bound = 1e-4 + 2 * (ev[-1] / ev[0]) * rel_fro(HXr, ref["HX_rot"])
    assert rel_fro(Ug, ref["U_c"]) <= bound, (rel_fro(Ug, ref["U_c"]), bound)
    codes = res.codes.cpu().numpy()
    same = (codes == ref["codes"]).mean()
    assert same >= 0.999, same
    # layer loss tr(H_G' dW' H_X' dW'^T): the GPU's own helper on its own outputs
    out = torch.zeros(1, dtype=torch.float64, device=cuda)
    abi.kronq_layer_loss(res.W_rot, res.W_hat, res.H_X, res.H_G, out,
                         abi.workspace(256, 256, device=cuda))
    assert abs(out.item() / ref["loss"] - 1) <= 0.01
    # packed words of the GPU codes are the oracle's packing of the same codes
    from oracle import pack as opack
    np.testing.assert_array_equal(res.packed.cpu().numpy().view(np.uint32), opack.pack(codes, 4))
    assert res.info.item() == 0


def test_shared_input_ranking_matches_oracle(cuda):
    """q/k/v-style sublayers on one input site: identical ranking by s, and
    the host allocation on the GPU scores equals the oracle's."""
    base = synth.get_config("toy-256")
    subs = tuple(synth.Sublayer(name, m, 256, "in", i, None, -1)
                 for i, (name, m) in enumerate([("q", 256), ("k", 64), ("v", 64), ("o", 256)]))
    cfg = dataclasses.replace(base, sublayers=subs)
    HX = opipe.x_covariance(cfg, cfg.sites[0])
    s_gpu, s_ref = [], []
    for sub in subs:
        _, _, res = _gpu_layer(cfg, sub, cuda, 4, keep=False)
        s_gpu.append(res.sens[0].item())
        HG = opipe.g_covariance(cfg, sub)
        s_ref.append(opipe.quantize_sublayer(cfg, sub, HX, HG, 4, rows=np.arange(2))["s"])
    assert osens.ranking(s_gpu) == osens.ranking(s_ref)
    params = [s.m * s.n for s in subs]
    assert alloc.allocate_bits(s_gpu, params, 3.0) == osens.allocate_bits(s_ref, params, 3.0)
    np.testing.assert_allclose(s_gpu, s_ref, rtol=1e-4)
