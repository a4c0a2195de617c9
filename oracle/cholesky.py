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
