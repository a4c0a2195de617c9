"""Incoherence diagnostics (fp64), for measurement only.

KronQ summary (hyper.ai), "Method", and the review's Figure 2 caption: the
incoherence measure mu(H)/sqrt(d) of H_G is close to 1 before processing and
drops below 0.10 after it; BiIP lowers the coefficient of variation of both
the column norms (CV_in) and the row norms (CV_out) of W, where input-side
processing alone leaves CV_out nearly unchanged.

Readings (the pages name the measures without formulas):
  * mu-incoherence as in the incoherence-processing literature the pages
    build on: H = Q diag(lambda) Q^T is mu-incoherent when
    max_ij |Q_ij| <= mu / sqrt(d), so mu(H) / sqrt(d) = max_ij |Q_ij|
    (1 for a diagonal H, 1/sqrt(d) at best).
  * CV = standard deviation / mean of the L2 norms (population standard
    deviation), of the columns (CV_in) or of the rows (CV_out) of the weight
    matrix being quantized.
"""

from __future__ import annotations

import numpy as np


def mu_normalized(H: np.ndarray) -> float:
    """max |Q_ij| over the orthonormal eigenvectors Q of the symmetric H."""
    _, Q = np.linalg.eigh(np.asarray(H, dtype=np.float64))
    return float(np.max(np.abs(Q)))


def _cv(norms: np.ndarray) -> float:
    norms = np.asarray(norms, dtype=np.float64)
    mean = float(np.mean(norms))
    return float(np.std(norms) / mean) if mean > 0 else 0.0


def cv_in(W: np.ndarray) -> float:
    """Coefficient of variation of the column norms of W (m x n)."""
    W = np.asarray(W, dtype=np.float64)
    return _cv(np.sqrt((W * W).sum(axis=0)))


def cv_out(W: np.ndarray) -> float:
    """Coefficient of variation of the row norms of W (m x n)."""
    W = np.asarray(W, dtype=np.float64)
    return _cv(np.sqrt((W * W).sum(axis=1)))
