"""Randomized orthogonal transforms U = T_m D_u and V = T_n D_v (fp64).

KronQ summary (hyper.ai), "Method" (Eq. 12): U and V are randomized
Hadamard transforms; KronQ README (GitHub), "Reproduce from scratch":
``--incoh_kernel had``.

Reading for widths that are not powers of two (the pages are silent; the
LLaMA widths 11008 = 43 * 2^8, 14336 = 7 * 2^11, 28672 = 7 * 2^12 need it):
write d = q * 2^k with q odd and take

    T_d = C_q (x) (H_{2^k} / sqrt(2^k)),

where H_{2^k} is the Sylvester Hadamard matrix and C_q the orthonormal
DCT-II matrix of size q (C_1 = [1], so powers of two get the plain normalized
Hadamard matrix).  A vector of length d is read as q segments of 2^k
consecutive entries: each segment gets the Hadamard transform, then the
segments are mixed by C_q.  The random signs D act first: x -> T_d D x.
Only orthogonality is load-bearing for the method (Theorem 1).
"""

from __future__ import annotations

import numpy as np


def split_width(d: int):
    """d = q * 2^k with q odd; returns (q, k)."""
    if d <= 0:
        raise ValueError("width must be positive")
    k = 0
    while d % 2 == 0:
        d //= 2
        k += 1
    return d, k


def sylvester(k: int) -> np.ndarray:
    """H_{2^k} from H_1 = [1], H_{2n} = [[H_n, H_n], [H_n, -H_n]] (unnormalized)."""
    H = np.ones((1, 1))
    for _ in range(k):
        H = np.block([[H, H], [H, -H]])
    return H


def fwht(x: np.ndarray) -> np.ndarray:
    """Unnormalized Walsh-Hadamard transform along the last axis (Sylvester
    order), by the recursive butterfly: for h = 1, 2, 4, ..., pairs
    (i, i + h) inside each block of 2h become (a + b, a - b)."""
    x = np.array(x, dtype=np.float64, copy=True)
    n = x.shape[-1]
    if n & (n - 1):
        raise ValueError("fwht length must be a power of two")
    h = 1
    while h < n:
        y = x.reshape(x.shape[:-1] + (n // (2 * h), 2, h))
        a = y[..., 0, :].copy()
        b = y[..., 1, :]
        y[..., 0, :] = a + b
        y[..., 1, :] = a - b
        x = y.reshape(x.shape)
        h *= 2
    return x


def dct2(q: int) -> np.ndarray:
    """Orthonormal DCT-II: C[p, s] = sqrt(2/q) c_p cos(pi (2 s + 1) p / (2 q)),
    c_0 = 1/sqrt(2), c_p = 1 otherwise."""
    p = np.arange(q)[:, None]
    s = np.arange(q)[None, :]
    C = np.sqrt(2.0 / q) * np.cos(np.pi * (2 * s + 1) * p / (2 * q))
    C[0, :] *= 1.0 / np.sqrt(2.0)
    return C


def dense(d: int, signs: np.ndarray | None = None) -> np.ndarray:
    """The d x d matrix T_d D (D = diag(signs), identity when signs is None)."""
    q, k = split_width(d)
    T = np.kron(dct2(q), sylvester(k) / np.sqrt(2.0 ** k))
    if signs is not None:
        T = T * np.asarray(signs, dtype=np.float64)[None, :]
    return T


def apply(x: np.ndarray, signs: np.ndarray | None = None) -> np.ndarray:
    """y = T_d D x for every vector along the last axis of x."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    q, k = split_width(d)
    if signs is not None:
        x = x * np.asarray(signs, dtype=np.float64)
    y = fwht(x.reshape(x.shape[:-1] + (q, 2 ** k))) / np.sqrt(2.0 ** k)
    if q > 1:
        y = np.einsum("ps,...sr->...pr", dct2(q), y)
    return y.reshape(x.shape)


def apply_t(y: np.ndarray, signs: np.ndarray | None = None) -> np.ndarray:
    """x = (T_d D)^T y = D T_d^T y along the last axis (the exact inverse)."""
    y = np.asarray(y, dtype=np.float64)
    d = y.shape[-1]
    q, k = split_width(d)
    z = y.reshape(y.shape[:-1] + (q, 2 ** k))
    if q > 1:
        z = np.einsum("sp,...sr->...pr", dct2(q), z)
    x = fwht(z) / np.sqrt(2.0 ** k)
    x = x.reshape(y.shape)
    if signs is not None:
        x = x * np.asarray(signs, dtype=np.float64)
    return x


def rows(d: int, idx, signs: np.ndarray | None = None) -> np.ndarray:
    """Rows idx of the d x d matrix T_d D, without forming it: row i is
    (T_d D)^T e_i, i.e. apply_t of the i-th unit vector."""
    idx = np.asarray(idx, dtype=np.int64)
    E = np.zeros((len(idx), d))
    E[np.arange(len(idx)), idx] = 1.0
    return apply_t(E, signs)
