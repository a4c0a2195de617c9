"""Whole-chain parity at full size on the LLaMA-2-7B-shaped q_proj layer
(W 4096 x 4096, X and G 262144 x 4096 bf16, W4 asymmetric per-channel,
BiIP, 1 % damping): both sides start from the same seeded inputs and each
computes every step itself -- the GPU through the C ABI in the order the
benchmark runs it, the fp64 oracle with its own covariances over all
262144 tokens, its own rescale and rotations, its own damped inverse
Cholesky factor and the unblocked column loop on every row.  Nothing of the
GPU's intermediate results reaches the oracle.

KronQ summary (hyper.ai), "Method" (Eq. 7 covariances, Eqs. 11-12 BiIP,
Eq. 14 sensitivity, Prop. 1 column update); KronQ review (pith.science),
appendix, Algorithms 1-2.

Bars: H_X, H_G <= 1e-4 relative Frobenius; >= 99.9 % identical
codes; the layer loss tr(H_G' dW' H_X' dW'^T) within 1 %; packed words
bit-exact where the codes are identical.  Intermediate stages carry the
differences of the stages before them, so their bars are derived: a
relative input error eps moves S = (H_jj / ||W_j||^2)^alpha by about
alpha eps, the orthogonal rotations keep relative errors, and the inverse
Cholesky factor of the damped matrix moves by at most about
kappa(H_d) eps (first-order perturbation of the factorisation), with
kappa(H_d) computed here.  U_c is also checked stage-isolated (the oracle
factors the GPU's own H_X') at the 1e-4 bar.
"""

from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import synth
from gpu_helpers import rel_fro, t
from oracle import cholesky as ochol
from oracle import pack as opack
from oracle import pipeline as opipe
from oracle import quantizer as oq
from post_quantization_02_b200 import pipeline as gpipe

pytestmark = pytest.mark.gpu


def _draw(chunk_fn, tokens, width, dev):
    """Each seeded chunk drawn once: copied to the device (the GPU's input)
    and accumulated by the oracle in fp64 over the exact bf16 values.
    Returns (A on the device, the oracle's A^T A / N)."""
    A = torch.empty((tokens, width), dtype=torch.bfloat16, device=dev)
    H = np.zeros((width, width))
    nch = synth.n_chunks(tokens)
    threads = max(1, min(16, os.cpu_count() or 1))
    with ThreadPoolExecutor(threads) as ex:
        for c0 in range(0, nch, threads):
            parts = list(ex.map(chunk_fn, range(c0, min(nch, c0 + threads))))
            for c, bits in zip(range(c0, nch), parts):
                r0 = c * synth.CHUNK_TOKENS
                A[r0:r0 + bits.shape[0]].copy_(
                    torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16))
                C = synth.bf16_bits_to_f32(bits).astype(np.float64)
                H += C.T @ C
    return A, H / tokens


def test_llama2_7b_q_proj_full_chain(cuda):
    cfg = synth.get_config("llama2-7b-q_proj")
    sub = cfg.sublayers[0]
    site = cfg.site(sub.site)
    N, m, n, bits = cfg.tokens, sub.m, sub.n, sub.bits

    # ---- inputs, the GPU's covariances (one launch each) and the oracle's
    X, hx = _draw(lambda c: synth.x_chunk(cfg, site, c), N, n, cuda)
    HXg = gpipe.covariance(X)
    del X
    G, hg = _draw(lambda c: synth.g_chunk(cfg, sub, c), N, m, cuda)
    HGg = gpipe.covariance(G)
    del G
    torch.cuda.empty_cache()
    assert rel_fro(HXg.cpu().numpy(), hx) <= 1e-4
    assert rel_fro(HGg.cpu().numpy(), hg) <= 1e-4

    # ---- the rest of the GPU chain: BiIP, s, inverse Cholesky, solver, pack
    su, sv = synth.make_signs(cfg, sub)
    res = gpipe.quantize_sublayer(t(synth.make_w(cfg, sub), cuda), HXg, HGg, t(su, cuda),
                                  t(sv, cuda), bits, sub.group, cfg.alpha, cfg.mode, cfg.damp,
                                  cfg.block, keep=True)
    torch.cuda.synchronize()
    assert res.info.item() == 0

    # ---- the oracle's own chain on every row
    ref = opipe.quantize_sublayer(cfg, sub, hx, hg, bits, loop="c")
    eps_h = max(rel_fro(HXg.cpu().numpy(), hx), rel_fro(HGg.cpu().numpy(), hg))

    # BiIP and s
    np.testing.assert_allclose(res.S_X.cpu().numpy(), ref["S_X"], rtol=1e-4)
    np.testing.assert_allclose(res.S_G.cpu().numpy(), ref["S_G"], rtol=1e-4)
    HXr = res.H_X.cpu().numpy()
    assert rel_fro(res.W_rot.cpu().numpy(), ref["W_rot"]) <= 1e-4
    assert rel_fro(HXr, ref["HX_rot"]) <= 1e-4
    assert rel_fro(res.H_G.cpu().numpy(), ref["HG_rot"]) <= 1e-4
    np.testing.assert_allclose(res.sens[0].item(), ref["s"], rtol=1e-4)

    # inverse Cholesky: stage-isolated at 1e-4, end to end within the
    # perturbation bound kappa(H_d) * eps of its input
    Ug = res.U_c.cpu().numpy()
    assert rel_fro(Ug, ochol.inverse_cholesky(ochol.damp(HXr, cfg.damp))) <= 1e-4
    Hd = ochol.damp(ref["HX_rot"], cfg.damp)
    ev = np.linalg.eigvalsh(Hd)
    kappa = ev[-1] / ev[0]
    eps_in = rel_fro(HXr, ref["HX_rot"])
    assert rel_fro(Ug, ref["U_c"]) <= 1e-4 + 2 * kappa * eps_in, (rel_fro(Ug, ref["U_c"]), kappa)

    # solver: codes, grids, loss
    codes = res.codes.cpu().numpy()
    same = (codes == ref["codes"]).mean()
    assert same >= 0.999, same
    np.testing.assert_allclose(res.scales.cpu().numpy(), ref["scale"], rtol=1e-4)
    assert (res.zeros.cpu().numpy() == ref["zero"]).mean() >= 0.999
    loss_gpu = oq.layer_loss(res.W_rot.cpu().numpy() - res.W_hat.cpu().numpy(), ref["HX_rot"],
                             ref["HG_rot"])
    assert abs(loss_gpu / ref["loss"] - 1) <= 0.01, (loss_gpu, ref["loss"])

    # packing: the GPU's words are the packing of its codes, and equal the
    # oracle's words on every row whose codes are identical
    pg = res.packed.cpu().numpy().view(np.uint32)
    np.testing.assert_array_equal(pg, opack.pack(codes, bits))
    rows = (codes == ref["codes"]).all(axis=1)
    np.testing.assert_array_equal(pg[rows], ref["packed"][rows])
    print(f"full chain: H rel err {eps_h:.2e}, kappa(H_d) {kappa:.1f}, identical codes "
          f"{same * 100:.3f} %, loss ratio {loss_gpu / ref['loss']:.6f}")
