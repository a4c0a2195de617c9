"""GPTAQ asymmetric calibration inside the KronQ column loop (fp64).

Test infrastructure: only tests/, the smoke check and the benchmark's CPU
baseline use this package.

Sources:
  * KronQ summary (hyper.ai), "Method": building on GPTAQ, the objective is
    corrected for input drift by asymmetric calibration -- the quantized
    layer sees X~ (the input the partly quantized model produces) while its
    target is the full-precision W X; the weight compensation after
    quantizing column p is written with the scaled error delta_p and "the
    GPTAQ asymmetric correction matrix" P (the display equation itself is
    lost from the page).
  * KronQ review (pith.science), appendix, Algorithm 2: inputs H_X,
    Delta X X^T, S_X, S_G, U, V from Algorithm 1; step 1 damping; step 2
    L <- InverseCholesky(H_X); step 3 P <- alpha (Delta X X^T L) (.) M_U L^T
    with M_U the upper-triangular mask; then the column loop in blocks.
  * GPTAQ (Li et al., 2025, "Efficient finetuning-free quantization for
    asymmetric calibration"), which the pages cite as the solver's origin.

Readings (the pages leave these open):
  * Delta X = X - X~ (full-precision input minus the drifted input) and
    Delta X X^T = (1/N) sum_t (x_t - x~_t) x~_t^T over the calibration
    tokens; H_X = (1/N) sum_t x~_t x~_t^T (the solver's Hessian is taken on
    the inputs the quantized layer actually sees).
  * BiIP acts on Delta X X^T as on H_X: both are products of input-side
    vectors, so Delta X X^T -> V S_X^-1 (Delta X X^T) S_X^-1 V^T with the
    S_X and V of H_X.
  * L is the lower Cholesky factor of the damped H_X^-1 (H_X^-1 = L L^T),
    i.e. U_c^T for the upper factor U_c the column update reads; M_U keeps
    the diagonal.  Row p of P / alpha is then the damped least-squares
    regression of input channel p's drift onto channels p, p+1, ... of X~
    (pinned in the tests).
  * The compensation after quantizing column p: every later column k > p
    receives -delta_p U_c[p, k] + w_p P[p, k], where w_p is column p's
    current value (the value the quantizer saw) -- the in-place column loop
    of Algorithm 2 holding W, with P's row p weighted by the column it was
    built for.
  * alpha is GPTAQ's scaling of P (Algorithm 2's "scaling alpha"), separate
    from the BiIP exponent; 0.25 unless given.
"""

from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from . import quantizer
from . import transform


def drift_covariance(X: np.ndarray, Xq: np.ndarray) -> np.ndarray:
    """(1/N) sum_t (x_t - x~_t) x~_t^T for token-major X, X~ (N x n), fp64."""
    X = np.asarray(X, dtype=np.float64)
    Xq = np.asarray(Xq, dtype=np.float64)
    N = X.shape[0]
    return (X - Xq).T @ Xq / N if N else np.zeros((X.shape[1], X.shape[1]))


def rotate_like_hx(A: np.ndarray, SX: np.ndarray, sign_v: np.ndarray, rotate: bool = True):
    """V S_X^-1 A S_X^-1 V^T (V = T_n D_v), the input-side BiIP of H_X
    applied to any n x n matrix built from input-side vectors."""
    A = np.asarray(A, dtype=np.float64) / np.asarray(SX, dtype=np.float64)[:, None]
    A = A / np.asarray(SX, dtype=np.float64)[None, :]
    if rotate:
        A = transform.apply(A, sign_v)             # A V^T: the transform along rows
        A = transform.apply(A.T, sign_v).T         # V (A V^T)
    return A


def correction(A: np.ndarray, U: np.ndarray, alpha: float = 0.25) -> np.ndarray:
    """P = alpha ((Delta X X^T L) (.) M_U) L^T with L = U^T (H_X^-1 = L L^T),
    M_U the upper-triangular mask with its diagonal (Algorithm 2, step 3)."""
    L = np.asarray(U, dtype=np.float64).T
    T = np.asarray(A, dtype=np.float64) @ L
    return alpha * (np.triu(T) @ L.T)


def obs_quantize_gptaq(W: np.ndarray, U: np.ndarray, P: np.ndarray, bits: int, group: int = -1):
    """The unblocked column loop of obs_quantize with the GPTAQ term: after
    column j is quantized, every later column k receives
    -e_j U[j, k] + v_j P[j, k] (v_j: column j's value the quantizer saw)."""
    W = np.array(W, dtype=np.float64)
    U = np.asarray(U, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    m, n = W.shape
    quantizer._check(n, group, bits)
    ng = 1 if group == -1 else n // group
    codes = np.zeros((m, n), dtype=np.uint8)
    scales = np.zeros((m, ng), dtype=np.float32)
    zeros = np.zeros((m, ng), dtype=np.uint8)
    What = np.zeros((m, n))
    if group == -1:
        scale, zero = quantizer.grid_params(W, bits)
        scales[:, 0], zeros[:, 0] = scale, zero
    for j in range(n):
        if group != -1 and j % group == 0:
            scale, zero = quantizer.grid_params(W[:, j:j + group], bits)
            scales[:, j // group], zeros[:, j // group] = scale, zero
        v = W[:, j].copy()
        q = quantizer.quantize(v, scale, zero, bits)
        wh = quantizer.dequantize(q, scale, zero)
        e = (v - wh) / U[j, j]
        W[:, j + 1:] -= np.outer(e, U[j, j + 1:])
        W[:, j + 1:] += np.outer(v, P[j, j + 1:])
        codes[:, j] = q
        What[:, j] = wh
    return {"codes": codes, "scale": scales, "zero": zeros, "W_hat": What}


def asymmetric_loss(W_hat: np.ndarray, W: np.ndarray, X: np.ndarray, Xq: np.ndarray) -> float:
    """(1/N) sum_t ||W_hat x~_t - W x_t||^2 (token-major X, X~): the
    objective the asymmetric calibration targets."""
    R = np.asarray(Xq, dtype=np.float64) @ np.asarray(W_hat, dtype=np.float64).T \
        - np.asarray(X, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T
    return float(np.sum(R * R) / max(1, R.shape[0]))


def obs_quantize_gptaq_rows(W: np.ndarray, U: np.ndarray, P: np.ndarray, bits: int,
                            group: int = -1, rows=None, chunk: int = 32,
                            threads: int | None = None):
    """obs_quantize_gptaq on a subset of rows, in row chunks on a thread pool
    (the loop treats rows independently, so this changes no operation)."""
    W = np.asarray(W)
    rows = np.arange(W.shape[0]) if rows is None else np.asarray(rows)
    parts = [rows[i:i + chunk] for i in range(0, len(rows), chunk)]
    threads = threads or min(32, os.cpu_count() or 1)
    U = np.asarray(U, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    with ThreadPoolExecutor(threads) as ex:
        res = list(ex.map(lambda r: obs_quantize_gptaq(W[r], U, P, bits, group), parts))
    return {k: np.concatenate([r[k] for r in res], axis=0) for k in res[0]}


def chain(cfg, sub, X_bits, Xq_bits, G_bits, bits, alpha_asym: float = 0.25, rows=None):
    """The whole fp64 chain of one sublayer with the asymmetric calibration,
    from the token-major bf16 inputs X, X~, G: H~ = X~^T X~ / N, the drift
    covariance, H_G, BiIP, the drift covariance rotated like H~, the damped
    inverse Cholesky factor, P, the column loop with the P term."""
    import synth
    from . import biip as _biip, cholesky, quantizer as _q
    X = synth.bf16_bits_to_f32(X_bits).astype(np.float64)
    Xq = synth.bf16_bits_to_f32(Xq_bits).astype(np.float64)
    Gm = synth.bf16_bits_to_f32(G_bits).astype(np.float64)
    N = X.shape[0]
    HX = Xq.T @ Xq / N
    A = drift_covariance(X, Xq)
    HG = Gm.T @ Gm / N
    W = synth.make_w(cfg, sub)
    su, sv = synth.make_signs(cfg, sub)
    Wp, HXt, HGt, SX, SG = _biip.biip(W, HX, HG, su, sv, cfg.alpha, cfg.mode)
    At = rotate_like_hx(A, SX, sv, rotate=cfg.mode != "su_only")
    U = cholesky.inverse_cholesky(cholesky.damp(HXt, cfg.damp))
    P = correction(At, U, alpha_asym)
    res = obs_quantize_gptaq_rows(Wp, U, P, bits, sub.group, rows=rows)
    out = {"HX": HX, "A": A, "HG": HG, "W_rot": Wp, "HX_rot": HXt, "HG_rot": HGt, "A_rot": At,
           "S_X": SX, "S_G": SG, "U_c": U, "P": P}
    out.update(res)
    if rows is None:
        out["loss"] = _q.layer_loss(Wp - res["W_hat"], HXt, HGt)
    return out
