"""Kronecker factors H_X = E[x x^T] and H_G = E[g g^T] (fp64).

KronQ summary (hyper.ai), "Method": for y = W x the per-sample gradient is
dL/dW = g x^T; the empirical Fisher is E[vec(g x^T) vec(g x^T)^T]; with x
independent of g it factorises as H_X (x) H_G, H_X = E[x x^T], H_G = E[g g^T]
(Eq. 7).  The expectation over the calibration set is the mean over its N
tokens (a reading: the pages write E[.] and calibrate on 128 x 2048 tokens).
"""

from __future__ import annotations

import numpy as np


def covariance(A: np.ndarray) -> np.ndarray:
    """(1/N) sum_t a_t a_t^T for the N rows a_t of A (N x d), in fp64."""
    A = np.asarray(A, dtype=np.float64)
    N = A.shape[0]
    if N == 0:
        return np.zeros((A.shape[1], A.shape[1]))
    return (A.T @ A) / N


def covariance_stream(chunks, d: int, n_total: int) -> np.ndarray:
    """Same mean, accumulated over row chunks (each chunk N_c x d)."""
    H = np.zeros((d, d))
    for C in chunks:
        C = np.asarray(C, dtype=np.float64)
        H += C.T @ C
    return H / n_total


def covariance_block(chunks, rows: np.ndarray, cols: np.ndarray, n_total: int) -> np.ndarray:
    """The sub-block H[rows][:, cols] only, over row chunks of A."""
    H = np.zeros((len(rows), len(cols)))
    for C in chunks:
        C = np.asarray(C, dtype=np.float64)
        H += C[:, rows].T @ C[:, cols]
    return H / n_total


def covariance_diag(chunks, d: int, n_total: int) -> np.ndarray:
    """diag(H) = (1/N) sum_t a_t[j]^2 for every j, over row chunks of A."""
    s = np.zeros(d)
    for C in chunks:
        C = np.asarray(C, dtype=np.float64)
        s += np.einsum("tj,tj->j", C, C)
    return s / n_total


def vec(M: np.ndarray) -> np.ndarray:
    """Column-stacking vec: vec(g x^T) = x (x) g."""
    return np.asarray(M).reshape(-1, order="F")


def empirical_fisher(xs, gs) -> np.ndarray:
    """Brute-force E[vec(g x^T) vec(g x^T)^T] over paired samples (x_t, g_t)."""
    acc = None
    for x, g in zip(xs, gs):
        v = vec(np.outer(g, x))
        o = np.outer(v, v)
        acc = o if acc is None else acc + o
    return acc / len(xs)


def kfac(HX: np.ndarray, HG: np.ndarray) -> np.ndarray:
    """H ~ H_X (x) H_G under the column-stacking vec of W (m x n)."""
    return np.kron(HX, HG)
