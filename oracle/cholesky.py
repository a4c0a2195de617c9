"""Damping and the inverse Cholesky factor (fp64).

KronQ review (pith.science), appendix, Algorithm 2 (KronQ quantization loop):
step 1 damps H_X <- H_X + lambda * mean(diag(H_X)) I; step 2 takes
L <- InverseCholesky(H_X).

Reading of "InverseCholesky": the upper-triangular U with
H^-1 = U^T U and a positive diagonal (the factor the column loop reads row by
row: the error of column j divides by U[j, j] and propagates along U[j, j:]).
The oracle forms H^-1 from a Cholesky factor of H by two triangular solves,
then takes the upper Cholesky factor of H^-1: the plain definition.
lambda multiplies the mean of the diagonal of the matrix handed to the
solver, i.e. of the rotated H_X (Algorithm 2 takes H_X from Algorithm 1).
"""

from __future__ import annotations

import numpy as np
import scipy.linalg as sla


class NotPositiveDefinite(ValueError):
    pass


def damp(H: np.ndarray, lam: float) -> np.ndarray:
    H = np.array(H, dtype=np.float64)
    n = H.shape[0]
    if n == 0:
        return H
    mu = float(np.mean(np.diag(H)))
    H[np.arange(n), np.arange(n)] += lam * mu
    return H


def inverse_cholesky(H: np.ndarray) -> np.ndarray:
    """Upper U with U^T U = H^-1 (H symmetric positive definite)."""
    H = np.asarray(H, dtype=np.float64)
    n = H.shape[0]
    try:
        L = np.linalg.cholesky(H)
    except np.linalg.LinAlgError as e:
        raise NotPositiveDefinite(str(e)) from None
    Linv = sla.solve_triangular(L, np.eye(n), lower=True)
    Hinv = Linv.T @ Linv
    Hinv = 0.5 * (Hinv + Hinv.T)
    try:
        Lh = np.linalg.cholesky(Hinv)
    except np.linalg.LinAlgError as e:
        raise NotPositiveDefinite(str(e)) from None
    return Lh.T


def inverse_cholesky_trailing(H: np.ndarray, k: int, lam: float = 0.0) -> np.ndarray:
    """U[k:, k:] of U = inverse_cholesky(damp(H, lam)), from H[k:, k:] and the
    mean of diag(H) alone.

    With R = U^-1 (upper), H_d = R R^T, and since R is upper the trailing
    block obeys H_d[k:, k:] = R[k:, k:] R[k:, k:]^T; the inverse of an upper
    triangular matrix has the inverse of its trailing block as its own
    trailing block, so U[k:, k:] = inverse_cholesky(H_d[k:, k:]).  The
    damping adds lam * mean(diag(H)) of the WHOLE matrix.  Lets a test check
    a wide factor on its last columns without the n^3 inverse."""
    H = np.asarray(H)
    n = H.shape[0]
    mu = float(np.mean(np.diag(H).astype(np.float64))) if n else 0.0
    B = np.array(H[k:, k:], dtype=np.float64)
    B[np.arange(n - k), np.arange(n - k)] += lam * mu
    return inverse_cholesky(B)
