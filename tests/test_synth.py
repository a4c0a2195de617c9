"""The seeded input generator: determinism, chunk independence, bf16
rounding and the distributions the configs state."""

import numpy as np
import torch

import synth
from synth.gen import outlier_channels, g_scales


def test_bf16_rounding_matches_torch():
    r = np.random.default_rng(0)
    x = (r.standard_normal(100000) * np.exp(r.uniform(-20, 20, 100000))).astype(np.float32)
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0]   # ties
    ours = synth.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = synth.bf16_bits_to_f32(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_chunks_are_independent_and_deterministic():
    cfg = synth.get_config("toy-256")
    site = cfg.sites[0]
    X = synth.make_x(cfg, site, tokens=40000, threads=3)
    assert X.shape == (40000, 256) and X.dtype == np.uint16
    c2 = synth.x_chunk(cfg, site, 2, tokens=40000)
    np.testing.assert_array_equal(X[2 * synth.CHUNK_TOKENS:], c2)
    np.testing.assert_array_equal(synth.make_x(cfg, site, tokens=40000, threads=1), X)


def test_toy_distributions():
    cfg = synth.get_config("toy-256")
    site, sub = cfg.sites[0], cfg.sublayers[0]
    X = synth.bf16_bits_to_f32(synth.make_x(cfg, site)).astype(np.float64)
    oc = outlier_channels(cfg, site)
    assert len(oc) == 4
    var = X.var(axis=0)
    normal = np.setdiff1d(np.arange(256), oc)
    assert 0.8 < var[normal].mean() < 1.2
    assert 300 < var[oc].mean() < 500          # x20 -> variance x400
    G = synth.bf16_bits_to_f32(synth.make_g(cfg, sub)).astype(np.float64)
    sc = g_scales(cfg, sub)
    assert sc.min() >= 10 ** -3 and sc.max() <= 1.0
    ratio = G.std(axis=0) / sc
    assert 0.9 < ratio.mean() < 1.1
    W = synth.make_w(cfg, sub)
    rs = W.std(axis=1) / 0.02
    assert rs.min() > 0.35 and rs.max() < 2.6
    su, sv = synth.make_signs(cfg, sub)
    assert set(np.unique(su)) == {-1, 1} and sv.shape == (256,)


def test_t4_and_outlier_fraction():
    cfg = synth.get_config("llama2-7b-q_proj")
    site = cfg.sites[0]
    assert cfg.outlier_count(4096) == 20
    assert cfg.outlier_count(11008) == 55
    X = synth.bf16_bits_to_f32(synth.x_chunk(cfg, site, 0, tokens=4096)).astype(np.float64)
    oc = outlier_channels(cfg, site)
    normal = np.setdiff1d(np.arange(4096), oc)
    v = X[:, normal].var()
    assert 1.6 < v < 2.4                        # Student-t(4) has variance 2
    W = synth.make_w(cfg, cfg.sublayers[0])
    # bf16-representable fp32 values
    np.testing.assert_array_equal(synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(W)), W)
