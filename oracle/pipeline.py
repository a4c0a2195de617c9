"""The whole per-layer chain in the order the KronQ pages run it, fp64.

KronQ review (pith.science), appendix: Algorithm 1 returns W, H_X, S_X,
S_G, U, V after BiIP; Algorithm 2 damps, takes the inverse Cholesky factor
and runs the column loop.  KronQ summary (hyper.ai), "Method": H_X and H_G
from the calibration activations and one backward pass; s = tr(H_G) tr(H_X)
after BiIP (Eq. 14).

  1. H_X = X^T X / N per input site, H_G = G^T G / N per sublayer
  2. BiIP: rescale, then U W V^T, V H_X V^T, U H_G U^T
  3. s = tr(H_G') tr(H_X')
  4. H = H_X' + lambda mean(diag H_X') I;  U_c = upper factor of H^-1
  5. column-wise OBS on W' onto the asymmetric grid
  6. pack the codes (2- and 4-bit)
"""

from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

import synth
from . import biip as _biip
from . import cholesky, pack, quantizer, sensitivity


def _chunk_cov(chunk_bits: np.ndarray) -> np.ndarray:
    C = synth.bf16_bits_to_f32(chunk_bits).astype(np.float64)
    return C.T @ C


def _stream_cov(fn, nchunks: int, d: int, n_total: int, threads) -> np.ndarray:
    threads = threads or min(8, os.cpu_count() or 1)
    H = np.zeros((d, d))
    with ThreadPoolExecutor(threads) as ex:
        for part in ex.map(lambda c: _chunk_cov(fn(c)), range(nchunks)):
            H += part
    return H / n_total if n_total else H


def x_covariance(cfg, site, tokens=None, threads=None) -> np.ndarray:
    """H_X = X^T X / N for one input site, over the exact bf16 values."""
    tokens = cfg.tokens if tokens is None else tokens
    return _stream_cov(lambda c: synth.x_chunk(cfg, site, c, tokens), synth.n_chunks(tokens),
                       site.width, tokens, threads)


def g_covariance(cfg, sub, tokens=None, threads=None) -> np.ndarray:
    tokens = cfg.tokens if tokens is None else tokens
    return _stream_cov(lambda c: synth.g_chunk(cfg, sub, c, tokens), synth.n_chunks(tokens),
                       sub.m, tokens, threads)


def quantize_sublayer(cfg, sub, HX, HG, bits, rows=None, W=None, act_order=False, clip=False,
                      loop="numpy"):
    """Steps 2-6 for one sublayer given its two covariances.

    rows: the rows of W' to run the column loop on (all when None); the loop
    treats rows independently, so a subset gives those rows' exact results.
    act_order / clip: the README's --act_order and --w_clip (readings in
    oracle/quantizer.py).  loop="c": the column loop through its plain-C
    restatement (bit-identical results; no act_order / clip there)."""
    if W is None:
        W = synth.make_w(cfg, sub)
    su, sv = synth.make_signs(cfg, sub)
    Wp, HXt, HGt, SX, SG = _biip.biip(W, HX, HG, su, sv, cfg.alpha, cfg.mode)
    s = sensitivity.sensitivity(HXt, HGt)
    Hd = cholesky.damp(HXt, cfg.damp)
    if act_order:
        perm = quantizer.act_order_perm(HXt)
        res = quantizer.obs_quantize_act_order(Wp, Hd, perm, bits, sub.group, clip=clip, rows=rows)
        Uc = res.pop("U_perm")
    else:
        perm = None
        Uc = cholesky.inverse_cholesky(Hd)
        if loop == "c" and not clip:
            res = quantizer.obs_quantize_rows_c(Wp, Uc, bits, sub.group, rows=rows)
        else:
            res = quantizer.obs_quantize_rows(Wp, Uc, bits, sub.group, rows=rows, clip=clip)
    out = {"W_rot": Wp, "HX_rot": HXt, "HG_rot": HGt, "S_X": SX, "S_G": SG, "s": s,
           "U_c": Uc, "perm": perm, "rows": np.arange(sub.m) if rows is None else np.asarray(rows)}
    out.update(res)
    if bits in (2, 4):
        out["packed"] = pack.pack(res["codes"], bits)
    if rows is None:
        out["loss"] = quantizer.layer_loss(Wp - res["W_hat"], HXt, HGt)
    return out
