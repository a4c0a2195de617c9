"""Parity at the full workload sizes, in the launch configuration the
benchmark times: one covariance launch over all 262144 tokens per H, one
BiIP call, one inverse Cholesky and one solver call per sublayer.

The fp64 oracle cannot redo layers this wide in seconds, so it checks
sampled outputs, each computed from its definition on the same inputs:

* H_X, H_G (KronQ summary, Method, Eq. 7): every diagonal entry and a seeded
  principal block of 256 indices (spanning many 128 x 256 tiles and the last
  tile), summed over all tokens in fp64; relative Frobenius <= 1e-4.
* BiIP (Eqs. 11-12): S_X and S_G in full; 64 x 64 blocks of W', H_X' and
  H_G', from the GPU's own fp32 stage inputs (stage isolation).
* s = tr(H_G') tr(H_X') (Eq. 14) and, on the decoder block, the ranking and
  the 2/3/4-bit allocation, from the oracle's own covariance diagonals.
* inverse Cholesky (review, Algorithm 2, steps 1-2): the trailing 2048 x 2048
  block of U_c exactly (it depends on the trailing block of H only), and
  U_c^T U_c H_d = I on sampled columns.
* OBS (Prop. 1: rows are independent given U_c): a seeded subset of 1024
  rows (all rows of narrower layers) through the unblocked oracle loop (its
  plain-C restatement, bit-identical to the numpy loop); >= 99.9 % identical
  codes, equal grids, and the subset's loss within 1 %.
* packing: every word, bit-exact.
"""

from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import synth
from gpu_helpers import rel_fro
from oracle import biip as obiip
from oracle import cholesky as ochol
from oracle import covariance as ocov
from oracle import pack as opack
from oracle import quantizer as oq
from oracle import sensitivity as osens
from post_quantization_02_b200 import abi, alloc

pytestmark = pytest.mark.gpu

COV_TOL = 1e-4          # bf16 inputs, fp32 accumulation (the parity bar)
ROT_TOL = 1e-5          # fp32 butterflies: ~log2(d) roundings of 2^-24 each
CHOL_TOL = 1e-4         # fp32 factor of a 1 %-damped matrix
PROP_TOL = 1e-2         # U^T U H_d = I residual on sampled columns (conditioning-bound)


def _sample(r, d, k=192, tail=64):
    """Seeded sorted indices: k spread over [0, d) plus the last `tail`."""
    idx = set(r.choice(max(1, d - tail), min(k, max(1, d - tail)), replace=False).tolist())
    idx.update(range(max(0, d - tail), d))
    return np.array(sorted(idx))


def _stream_to_device(chunk_fn, tokens, width, dev, idx, threads=8):
    """Draw a token-major bf16 tensor chunk by chunk into device memory and
    accumulate, as the chunks pass, the oracle's fp64 diag(A^T A) and
    (A^T A)[idx][:, idx].  Returns (A on the device, diag / N, block / N)."""
    A = torch.empty((tokens, width), dtype=torch.bfloat16, device=dev)
    diag = np.zeros(width)
    blk = np.zeros((len(idx), len(idx)))
    nch = synth.n_chunks(tokens)
    with ThreadPoolExecutor(threads) as ex:
        for c0 in range(0, nch, threads):
            parts = list(ex.map(chunk_fn, range(c0, min(nch, c0 + threads))))
            for c, bits in zip(range(c0, nch), parts):
                r0 = c * synth.CHUNK_TOKENS
                A[r0:r0 + bits.shape[0]].copy_(
                    torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16))
                f = synth.bf16_bits_to_f32(bits)
                diag += ocov.covariance_diag((f[i:i + 2048] for i in range(0, len(f), 2048)),
                                             width, 1)
                blk += ocov.covariance_block([f[:, idx]], np.arange(len(idx)),
                                             np.arange(len(idx)), 1)
    return A, diag / tokens, blk / tokens


def _check_cov(H, diag_ref, blk_ref, idx):
    Hh = H[torch.as_tensor(idx, device=H.device)][:, torch.as_tensor(idx, device=H.device)]
    Hh = Hh.cpu().numpy()
    d = torch.diagonal(H).cpu().numpy()
    assert rel_fro(Hh, blk_ref) <= COV_TOL, rel_fro(Hh, blk_ref)
    np.testing.assert_allclose(d, diag_ref, rtol=COV_TOL)
    # the kernel writes both triangles: the sampled block is symmetric exactly
    assert np.array_equal(Hh, Hh.T)


def _rows_for(n):
    """Solver rows the oracle re-runs at every width: its unblocked fp64
    loop costs rows * n^2 / 2 updates (the C restatement runs about 1e10
    of them per second on the host's cores: tens of seconds at n = 28672)."""
    return 1024


def _sublayer_chain(cfg, sub, HX, HG, bits, r, rows=None, full_loss=False):
    """BiIP -> s -> inverse Cholesky -> OBS -> pack on the GPU for one sublayer,
    each stage checked against the oracle on that stage's GPU inputs.
    HX, HG: the sublayer's covariances on the device (rotated in place)."""
    dev = HX.device
    m, n, group = sub.m, sub.n, sub.group
    W = synth.make_w(cfg, sub)
    su, sv = synth.make_signs(cfg, sub)
    HX_in, HG_in = HX.cpu().numpy(), HG.cpu().numpy()
    Wd = torch.from_numpy(W).to(dev)
    SX = torch.empty(n, device=dev)
    SG = torch.empty(m, device=dev)
    ws = abi.workspace(m, n, bits, group, device=dev)
    abi.kronq_biip_rotate(Wd, HX, HG, torch.from_numpy(su).to(dev), torch.from_numpy(sv).to(dev),
                          cfg.alpha, cfg.mode, 0, SX, SG, ws)
    sens = torch.zeros(3, dtype=torch.float64, device=dev)
    abi.kronq_sensitivity(HX, HG, sens)

    # ---- BiIP: scales in full, 64 x 64 blocks of each output
    wr, hgi = (np.sort(r.choice(m, 64, replace=False)) for _ in range(2))
    wc, hxi = (np.sort(r.choice(n, 64, replace=False)) for _ in range(2))
    Wb, HXb, HGb, SXr, SGr = obiip.biip_entries(W, HX_in, HG_in, su, sv, cfg.alpha, cfg.mode,
                                                wr, wc, hxi, hgi)
    np.testing.assert_allclose(SX.cpu().numpy(), SXr, rtol=10 * ROT_TOL)
    np.testing.assert_allclose(SG.cpu().numpy(), SGr, rtol=10 * ROT_TOL)
    Wrot = Wd.cpu().numpy()
    assert rel_fro(Wrot[np.ix_(wr, wc)], Wb) <= ROT_TOL
    HXr = HX.cpu().numpy()
    assert rel_fro(HXr[np.ix_(hxi, hxi)], HXb) <= ROT_TOL
    assert rel_fro(HG.cpu().numpy()[np.ix_(hgi, hgi)], HGb) <= ROT_TOL
    s_ref = osens.sensitivity_from_diagonals(np.diag(HX_in), np.diag(HG_in), SXr, SGr)
    np.testing.assert_allclose(sens[0].item(), s_ref, rtol=ROT_TOL)
    del HX_in, HG_in

    # ---- inverse Cholesky of the damped rotated H_X
    U = torch.empty((n, n), device=dev)
    info = torch.zeros(1, dtype=torch.int32, device=dev)
    abi.kronq_cholesky_inv(HX, cfg.damp, U, info, ws)
    torch.cuda.synchronize()
    assert info.item() == 0
    assert torch.count_nonzero(torch.tril(U, -1)).item() == 0
    Uh = U.cpu().numpy()
    k = max(0, n - 2048)
    assert rel_fro(Uh[k:, k:], ochol.inverse_cholesky_trailing(HXr, k, cfg.damp)) <= CHOL_TOL
    J = np.sort(r.choice(n, 16, replace=False))
    mu = float(np.mean(np.diag(HXr).astype(np.float64)))
    B = HXr[:, J].astype(np.float64)
    B[J, np.arange(len(J))] += cfg.damp * mu
    UB = np.vstack([Uh[p:p + 2048].astype(np.float64) @ B for p in range(0, n, 2048)])
    UtUB = sum(Uh[p:p + 2048].T.astype(np.float64) @ UB[p:p + 2048] for p in range(0, n, 2048))
    I_J = np.zeros((n, len(J)))
    I_J[J, np.arange(len(J))] = 1.0
    assert rel_fro(UtUB, I_J) <= PROP_TOL, rel_fro(UtUB, I_J)

    # ---- OBS on a row subset (rows are independent given U_c)
    G = 1 if group == -1 else n // group
    codes = torch.empty((m, n), dtype=torch.uint8, device=dev)
    scales = torch.empty((m, G), device=dev)
    zeros = torch.empty((m, G), dtype=torch.uint8, device=dev)
    What = torch.empty((m, n), device=dev)
    abi.kronq_quantize_layer(Wd, U, bits, group, cfg.block, codes, scales, zeros, What, info, ws)
    torch.cuda.synchronize()
    assert info.item() == 0
    rows = np.sort(r.choice(m, min(m, rows or _rows_for(n)), replace=False))
    U64 = Uh.astype(np.float64)
    del Uh
    ref = oq.obs_quantize_rows_c(Wrot[rows], U64, bits, group)
    del U64
    cg = codes.cpu().numpy()
    same = (cg[rows] == ref["codes"]).mean()
    assert same >= 0.999, same
    sc, zr = scales.cpu().numpy()[rows], zeros.cpu().numpy()[rows]
    if group == -1:
        np.testing.assert_array_equal(sc, ref["scale"])
        np.testing.assert_array_equal(zr, ref["zero"])
    else:
        # group grids come from the already-updated weights: a code that
        # flipped earlier in the row (equally valid, fp order) moves every
        # later grid of that row, so grids are compared on the groups with no
        # differing code before them; those carry only the rounding of the
        # lazy updates (bf16 hi / lo products, ~2^-17 relative)
        assert (zr == ref["zero"]).mean() >= 0.999
        diff = cg[rows] != ref["codes"]
        first_diff = np.where(diff.any(axis=1), diff.argmax(axis=1), n)
        clean = np.arange(sc.shape[1])[None, :] * group < first_diff[:, None]
        assert clean.mean() >= 0.9
        assert (np.abs(sc / ref["scale"] - 1)[clean] <= 1e-5).mean() >= 0.999
    Wh = What.cpu().numpy()
    lg = oq.row_losses(Wrot[rows] - Wh[rows], HXr, cfg.damp).sum()
    lr = oq.row_losses(Wrot[rows] - ref["W_hat"], HXr, cfg.damp).sum()
    assert abs(lg / lr - 1) <= 0.01, (lg, lr)
    assert cg.max() <= 2 ** bits - 1

    # ---- packing: every word
    if bits in (2, 4):
        packed = torch.empty((m, abi.packed_words(n, bits)), dtype=torch.int32, device=dev)
        abi.kronq_pack(codes, bits, packed)
        np.testing.assert_array_equal(packed.cpu().numpy().view(np.uint32), opack.pack(cg, bits))

    out = {"s": sens[0].item(), "same": same}
    if full_loss and len(rows) == m:
        # the whole layer's loss tr(H_G' dW' H_X' dW'^T) with undamped rotated H's
        out["loss_gpu"] = oq.layer_loss(Wrot - Wh, HXr, HG.cpu().numpy())
        out["loss_ref"] = oq.layer_loss(Wrot - ref["W_hat"], HXr, HG.cpu().numpy())
        out["rows"] = rows
        out["ref_codes"] = ref["codes"]
    return out


def _covariances(cfg, dev, r, sites=None, subs=None):
    """The configuration's covariances on the GPU (one launch each, as timed),
    each checked on its sampled entries; returns ({site: H_X}, {sub: H_G},
    {site: oracle diag}, {sub: oracle diag})."""
    N = cfg.tokens
    HX, HG, dx, dg = {}, {}, {}, {}
    for site in cfg.sites if sites is None else sites:
        idx = _sample(r, site.width)
        A, dref, bref = _stream_to_device(lambda c: synth.x_chunk(cfg, site, c), N, site.width,
                                          dev, idx)
        H = torch.empty((site.width, site.width), device=dev)
        abi.kronq_covariance(A, H, 1.0 / N, 0.0)
        del A
        _check_cov(H, dref, bref, idx)
        HX[site.name], dx[site.name] = H, dref
    for sub in cfg.sublayers if subs is None else subs:
        idx = _sample(r, sub.m)
        A, dref, bref = _stream_to_device(lambda c: synth.g_chunk(cfg, sub, c), N, sub.m, dev, idx)
        H = torch.empty((sub.m, sub.m), device=dev)
        abi.kronq_covariance(A, H, 1.0 / N, 0.0)
        del A
        _check_cov(H, dref, bref, idx)
        HG[sub.name], dg[sub.name] = H, dref
    torch.cuda.empty_cache()
    return HX, HG, dx, dg


def test_llama2_7b_q_proj_full_size(cuda):
    """The benchmarked layer: 4096 x 4096, W4 per-channel, 262144 tokens.
    The oracle re-runs the column loop on every row, so the whole layer's
    codes and its loss tr(H_G' dW' H_X' dW'^T) are compared."""
    cfg = synth.get_config("llama2-7b-q_proj")
    r = np.random.default_rng(101)
    HX, HG, _, _ = _covariances(cfg, cuda, r)
    sub = cfg.sublayers[0]
    out = _sublayer_chain(cfg, sub, HX[sub.site], HG[sub.name], sub.bits, r, rows=sub.m,
                          full_loss=True)
    assert out["same"] >= 0.999
    assert abs(out["loss_gpu"] / out["loss_ref"] - 1) <= 0.01


@pytest.mark.parametrize("name", ["gate_proj", "down_proj"])
def test_llama2_7b_mlp_full_size(cuda, name):
    """11008 x 4096 and 4096 x 11008 (odd factor 43), W2 group-128."""
    cfg = synth.get_config("llama2-7b-mlp")
    sub = next(s for s in cfg.sublayers if s.name == name)
    r = np.random.default_rng(202 + sub.index)
    HX, HG, _, _ = _covariances(cfg, cuda, r, sites=[cfg.site(sub.site)], subs=[sub])
    _sublayer_chain(cfg, sub, HX[sub.site], HG[sub.name], sub.bits, r)


@pytest.mark.parametrize("name", ["gate_proj", "down_proj"])
def test_llama3_70b_mlp_full_size(cuda, name):
    """28672 x 8192 and 8192 x 28672 (odd factor 7), W2 group-128: H_X of
    the down projection is 28672 x 28672 fp32 (3.3 GB) on one GPU."""
    cfg = synth.get_config("llama3-70b-mlp")
    sub = next(s for s in cfg.sublayers if s.name == name)
    r = np.random.default_rng(404 + sub.index)
    HX, HG, _, _ = _covariances(cfg, cuda, r, sites=[cfg.site(sub.site)], subs=[sub])
    _sublayer_chain(cfg, sub, HX[sub.site], HG[sub.name], sub.bits, r)


def test_llama3_8b_block_ranking_allocation_and_all_sublayers(cuda):
    """Seven sublayers on four input sites: every covariance at full size,
    s for each sublayer after BiIP, the ranking and the 2/3/4-bit allocation
    at a 3-bit average identical to the oracle's (whose s comes from its own
    fp64 covariance diagonals and its own S_X, S_G); then every sublayer
    through the rest of the chain at its allocated bits (3-bit codes stay
    unpacked)."""
    cfg = synth.get_config("llama3-8b-block")
    r = np.random.default_rng(303)
    HX, HG, dx, dg = _covariances(cfg, cuda, r)
    s_gpu, s_ref = [], []
    for sub in cfg.sublayers:
        W = synth.make_w(cfg, sub)
        su, sv = synth.make_signs(cfg, sub)
        hx = HX[sub.site].clone()
        hg = HG[sub.name].clone()
        Wd = torch.from_numpy(W).to(cuda)
        SX = torch.empty(sub.n, device=cuda)
        SG = torch.empty(sub.m, device=cuda)
        abi.kronq_biip_rotate(Wd, hx, hg, torch.from_numpy(su).to(cuda),
                              torch.from_numpy(sv).to(cuda), cfg.alpha, cfg.mode, 0, SX, SG,
                              abi.workspace(sub.m, sub.n, device=cuda))
        sens = torch.zeros(3, dtype=torch.float64, device=cuda)
        abi.kronq_sensitivity(hx, hg, sens)
        s_gpu.append(sens[0].item())
        SXr, SGr = obiip.scales(W, dx[sub.site], dg[sub.name], cfg.alpha, cfg.mode)
        s_ref.append(osens.sensitivity_from_diagonals(dx[sub.site], dg[sub.name], SXr, SGr))
        del hx, hg, Wd
    np.testing.assert_allclose(s_gpu, s_ref, rtol=COV_TOL)
    assert osens.ranking(s_gpu) == osens.ranking(s_ref)
    params = [s.m * s.n for s in cfg.sublayers]
    bits = alloc.allocate_bits(s_gpu, params, cfg.mixed_avg_bits)
    assert bits == osens.allocate_bits(s_ref, params, cfg.mixed_avg_bits)
    assert sorted(set(bits)) != [3], bits          # a real mix, not all 3-bit
    assert sum(b * p for b, p in zip(bits, params)) <= 3 * sum(params)
    # every sublayer through the rest of the chain, at its allocated bits; a
    # shared input site's H_X is rotated per sublayer, so each gets a copy
    for sub, b in zip(cfg.sublayers, bits):
        hx = HX[sub.site].clone()
        out = _sublayer_chain(cfg, sub, hx, HG.pop(sub.name), b, r)
        assert out["same"] >= 0.999
        del hx
        torch.cuda.empty_cache()


def test_llama2_7b_q_proj_act_order_and_clip_solver_full_size(cuda):
    """The README's --act_order and --w_clip (readings in include/kronq.h) on
    the benchmarked layer, in the launch sequence bench.py times with
    --act-order --w-clip: covariances -> BiIP -> act_order -> permute H_X',
    W' -> inverse Cholesky of the permuted damped H_X' -> solver with the
    clip search -> codes back to the original order.  Stage-isolated like
    the chain above: the oracle takes the GPU's fp32 H_X' and W' (so the
    permutation is compared bit-exact), factors the permuted damped matrix
    itself and re-runs the column loop on 1024 seeded rows."""
    cfg = synth.get_config("llama2-7b-q_proj")
    sub = cfg.sublayers[0]
    m, n, bits, group = sub.m, sub.n, sub.bits, sub.group
    r = np.random.default_rng(303)
    HXs, HGs, _, _ = _covariances(cfg, cuda, r)
    HX, HG = HXs[sub.site], HGs[sub.name]
    dev = cuda
    su, sv = synth.make_signs(cfg, sub)
    Wd = torch.from_numpy(synth.make_w(cfg, sub)).to(dev)
    ws = abi.workspace(m, n, bits, group, device=dev)
    SX, SG = torch.empty(n, device=dev), torch.empty(m, device=dev)
    abi.kronq_biip_rotate(Wd, HX, HG, torch.from_numpy(su).to(dev), torch.from_numpy(sv).to(dev),
                          cfg.alpha, cfg.mode, 0, SX, SG, ws)
    info = torch.zeros(1, dtype=torch.int32, device=dev)
    perm = torch.empty(n, dtype=torch.int32, device=dev)
    abi.kronq_act_order(HX, perm)
    Hp, Wp = torch.empty_like(HX), torch.empty_like(Wd)
    abi.kronq_permute(HX, Hp, perm, abi.PERM_SYM, info)
    abi.kronq_permute(Wd, Wp, perm, abi.PERM_COLS, info)
    U = torch.empty_like(HX)
    abi.kronq_cholesky_inv(Hp, cfg.damp, U, info, ws)
    cp = torch.empty((m, n), dtype=torch.uint8, device=dev)
    scales = torch.empty((m, 1), device=dev)
    zeros = torch.empty((m, 1), dtype=torch.uint8, device=dev)
    Whp = torch.empty((m, n), device=dev)
    abi.kronq_quantize_layer_opt(Wp, U, bits, group, cfg.block, abi.QUANT_CLIP, cp, scales, zeros,
                                 Whp, info, ws)
    codes, What = torch.empty_like(cp), torch.empty_like(Whp)
    abi.kronq_permute(cp, codes, perm, abi.UNPERM_COLS, info)
    abi.kronq_permute(Whp, What, perm, abi.UNPERM_COLS, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    HXr, Wrot = HX.cpu().numpy(), Wd.cpu().numpy()
    p_ref = oq.act_order_perm(HXr)
    np.testing.assert_array_equal(perm.cpu().numpy(), p_ref)
    rows = np.sort(r.choice(m, 1024, replace=False))
    Hd = ochol.damp(HXr, cfg.damp)
    ref = oq.obs_quantize_act_order(Wrot[rows], Hd, p_ref, bits, group, clip=True)
    cg = codes.cpu().numpy()[rows]
    same = (cg == ref["codes"]).mean()
    assert same >= 0.999, same
    np.testing.assert_array_equal(scales.cpu().numpy()[rows], ref["scale"])
    np.testing.assert_array_equal(zeros.cpu().numpy()[rows], ref["zero"])
    lg = oq.row_losses(Wrot[rows] - What.cpu().numpy()[rows], HXr, cfg.damp).sum()
    lr = oq.row_losses(Wrot[rows] - ref["W_hat"], HXr, cfg.damp).sum()
    assert abs(lg / lr - 1) <= 0.01, (lg, lr)
