"""Sensitivity score and the mixed-precision allocation.

KronQ summary (hyper.ai), "Method" (Eq. 14): the expected quantization loss
of sublayer l is proportional to eps_l^2 tr(H^(l)); with H ~ H_X (x) H_G,
tr(H) = tr(H_G) tr(H_X), and the score s_l = tr(H_G) tr(H_X) is computed
after BiIP; sublayers with larger s get more bits.  KronQ README (GitHub),
"Mapping paper results to flags": --inter_layer_mp N upgrades the top-N
sensitive sublayer types by +1 bit.

Reading for a 2/3/4-bit mix at a target average (the pages give the ranking
rule, not the budget rule): every sublayer starts at 2 bits; in descending
score order each one receives the largest upgrade (+2, else +1) that keeps
the parameter-weighted average at or below the target.  Equal scores keep
the decoder order q, k, v, o, gate, up, down (the sublayer index).
"""

from __future__ import annotations

import numpy as np


def sensitivity(HX: np.ndarray, HG: np.ndarray) -> float:
    """s = tr(H_G) * tr(H_X), summed in fp64."""
    return float(np.trace(np.asarray(HG, dtype=np.float64))) * \
        float(np.trace(np.asarray(HX, dtype=np.float64)))


def ranking(scores) -> list:
    """Indices by descending score; ties keep the lower index first."""
    scores = list(scores)
    return sorted(range(len(scores)), key=lambda i: (-scores[i], i))


def allocate_bits(scores, params, target_avg: float = 3.0, base: int = 2, top: int = 4) -> list:
    """Greedy 2/3/4 allocation (reading in the module docstring)."""
    params = [int(p) for p in params]
    total = sum(params)
    budget = int(round(target_avg * total))      # bits * params allowed in all
    bits = [base] * len(params)
    used = base * total
    for i in ranking(scores):
        for up in range(top - base, 0, -1):
            if used + up * params[i] <= budget:
                bits[i] += up
                used += up * params[i]
                break
    return bits


def sensitivity_from_diagonals(hx_diag, hg_diag, SX, SG) -> float:
    """The same s after BiIP, from the diagonals before it: the rotation is
    orthogonal, so tr(V H V^T) = tr(H), and the rescale divides entry j of
    the diagonal by S_j^2; hence s = (sum_j H_X[j,j] / S_X[j]^2) *
    (sum_i H_G[i,i] / S_G[i]^2), fp64.  Lets a test score a sublayer of any
    width without forming the rotated matrices."""
    tx = float(np.sum(np.asarray(hx_diag, dtype=np.float64) / np.asarray(SX, dtype=np.float64) ** 2))
    tg = float(np.sum(np.asarray(hg_diag, dtype=np.float64) / np.asarray(SG, dtype=np.float64) ** 2))
    return tg * tx
