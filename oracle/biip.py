"""Bidirectional incoherence processing (BiIP), fp64.

KronQ summary (hyper.ai), "Method": the input-side diagonal rescale is
extended to both column and row directions, the output-side S_G being new
(Eq. 11); then orthogonal transforms W' = U W V^T, H_G' = U H_G U^T,
H_X' = V H_X V^T with U, V randomized Hadamard transforms (Eq. 12).
KronQ review (pith.science), appendix A.2 (proof of Theorem 1): the loss
tr(H_G dW H_X dW^T) is unchanged by that transform.

Readings (Eq. 11 is missing from the extracted pages):
  * S_X[j] = (H_X[j, j] / ||W[:, j]||^2)^alpha from the original W; then
    W <- W diag(S_X), H_X <- S_X^-1 H_X S_X^-1.
  * S_G[i] = (H_G[i, i] / ||(W S_X)[i, :]||^2)^alpha from the column-scaled W;
    then W <- diag(S_G) W, H_G <- S_G^-1 H_G S_G^-1.
    Both keep the loss exactly invariant; at alpha = 1/4 each side equalises
    the rescaled diagonal with the rescaled squared norm.
  * A zero diagonal entry or a zero norm gives a scale of 1.  No global
    normalisation of S (it would change tr(H) and so the sensitivity score).
  * The rescale comes before the rotations ("subsequently, orthogonal
    transforms are applied").
  * --incoh_mode (KronQ README, "Mapping paper results to flags"):
    full = both rescales and both rotations; no_rescale = both rotations
    only; su_only = output side only (S_G and U); sv_only = input side only
    (S_X and V).
"""

from __future__ import annotations

import numpy as np

from . import transform

MODES = ("full", "no_rescale", "su_only", "sv_only")


def sides(mode: str):
    """(rescale input, rescale output, rotate input, rotate output)."""
    if mode == "full":
        return True, True, True, True
    if mode == "no_rescale":
        return False, False, True, True
    if mode == "su_only":
        return False, True, False, True
    if mode == "sv_only":
        return True, False, True, False
    raise ValueError(f"unknown incoherence mode {mode!r}")


def _scale(h_diag: np.ndarray, norm2: np.ndarray, alpha: float) -> np.ndarray:
    s = np.ones_like(h_diag, dtype=np.float64)
    ok = (h_diag > 0) & (norm2 > 0)
    s[ok] = (h_diag[ok] / norm2[ok]) ** alpha
    return s


def scales(W, hx_diag, hg_diag, alpha: float, mode: str = "full"):
    """S_X and S_G of Eq. 11 (reading above) from W and the two diagonals:
    S_X from the column norms of W, S_G from the row norms of W diag(S_X)."""
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    in_s, out_s, _, _ = sides(mode)
    SX = np.ones(n)
    SG = np.ones(m)
    if in_s:
        SX = _scale(np.array(hx_diag, dtype=np.float64), (W * W).sum(axis=0), alpha)
    if out_s:
        WS = W * SX[None, :]
        SG = _scale(np.array(hg_diag, dtype=np.float64), (WS * WS).sum(axis=1), alpha)
    return SX, SG


def rescale(W, HX, HG, alpha: float, mode: str = "full"):
    """Eq. 11 (reading above).  Returns W, H_X, H_G rescaled and S_X, S_G."""
    W = np.array(W, dtype=np.float64)
    HX = np.array(HX, dtype=np.float64)
    HG = np.array(HG, dtype=np.float64)
    SX, SG = scales(W, np.diag(HX), np.diag(HG), alpha, mode)
    W = W * SX[None, :] * SG[:, None]
    HX = HX / np.outer(SX, SX)
    HG = HG / np.outer(SG, SG)
    return W, HX, HG, SX, SG


def rotate(W, HX, HG, sign_u, sign_v, mode: str = "full"):
    """Eq. 12: W' = U W V^T, H_X' = V H_X V^T, H_G' = U H_G U^T."""
    W = np.asarray(W, dtype=np.float64)
    HX = np.asarray(HX, dtype=np.float64)
    HG = np.asarray(HG, dtype=np.float64)
    _, _, in_r, out_r = sides(mode)
    if in_r:
        W = transform.apply(W, sign_v)                          # rows: W V^T
        HX = transform.apply(transform.apply(HX.T, sign_v).T, sign_v)
    if out_r:
        W = transform.apply(W.T, sign_u).T                      # columns: U W
        HG = transform.apply(transform.apply(HG.T, sign_u).T, sign_u)
    return W, HX, HG


def biip(W, HX, HG, sign_u, sign_v, alpha: float = 0.25, mode: str = "full"):
    """Rescale then rotate.  Returns (W', H_X', H_G', S_X, S_G)."""
    W, HX, HG, SX, SG = rescale(W, HX, HG, alpha, mode)
    W, HX, HG = rotate(W, HX, HG, sign_u, sign_v, mode)
    return W, HX, HG, SX, SG


def unbiip_w(Wp, SX, SG, sign_u, sign_v, mode: str = "full"):
    """Exact inverse on W: W = S_G^-1 U^T W' V S_X^-1."""
    W = np.asarray(Wp, dtype=np.float64)
    _, _, in_r, out_r = sides(mode)
    if out_r:
        W = transform.apply_t(W.T, sign_u).T
    if in_r:
        W = transform.apply_t(W, sign_v)
    return W / np.asarray(SG)[:, None] / np.asarray(SX)[None, :]


def biip_entries(W, HX, HG, sign_u, sign_v, alpha: float, mode: str, w_rows, w_cols,
                 hx_idx, hg_idx):
    """Selected entries of the BiIP outputs at any size, without forming the
    whole transforms:
      W'[w_rows][:, w_cols]   = (U_r S_G) W (S_X V_c^T),
      H_X'[hx_idx][:, hx_idx] = V_a S_X^-1 H_X S_X^-1 V_a^T,
      H_G'[hg_idx][:, hg_idx] = U_a S_G^-1 H_G S_G^-1 U_a^T,
    where U_r, V_c, V_a, U_a are the selected rows of U = T_m D_u and
    V = T_n D_v (identity rows on a side the mode does not rotate).  The
    same products as rescale + rotate, associated so only the selected rows
    and columns are formed.  Returns (W' block, H_X' block, H_G' block,
    S_X, S_G); H_X / H_G may be None."""
    m, n = W.shape
    _, _, in_r, out_r = sides(mode)
    hxd = np.diag(HX) if HX is not None else np.ones(n)
    hgd = np.diag(HG) if HG is not None else np.ones(m)
    SX, SG = scales(W, hxd, hgd, alpha, mode)

    def sel(d, idx, signs, rot):
        if rot:
            return transform.rows(d, idx, signs)
        E = np.zeros((len(idx), d))
        E[np.arange(len(idx)), np.asarray(idx)] = 1.0
        return E

    def left(A, M, panel=2048):
        # A @ M with M widened to fp64 one row panel at a time (M may be a
        # wide fp32 matrix that would not fit in memory as fp64 at once)
        out = np.zeros((A.shape[0], M.shape[1]))
        for p in range(0, M.shape[0], panel):
            out += A[:, p:p + panel] @ np.asarray(M[p:p + panel], dtype=np.float64)
        return out

    Ur = sel(m, w_rows, sign_u, out_r) * SG[None, :]
    Vc = sel(n, w_cols, sign_v, in_r) * SX[None, :]
    Wb = left(Ur, W) @ Vc.T
    HXb = HGb = None
    if HX is not None:
        Va = sel(n, hx_idx, sign_v, in_r) / SX[None, :]
        HXb = left(Va, HX) @ Va.T
    if HG is not None:
        Ua = sel(m, hg_idx, sign_u, out_r) / SG[None, :]
        HGb = left(Ua, HG) @ Ua.T
    return Wb, HXb, HGb, SX, SG
