"""Deployment matvec of a quantized layer, fp64: y = W_hat x in the
original (unrotated, unscaled) space.

KronQ README (GitHub), deploy path: the packed int4 / int2 layer is served
by a kernel that dequantizes and applies the BiIP transforms online (fused
dequant + BiIP matvec, batch-1 decode).  KronQ summary (hyper.ai),
"Method" (Eqs. 11-12): W' = U S_G W S_X V^T, so the layer the codes stand
for is W_hat = S_G^-1 U^T W_hat' V S_X^-1, with W_hat' the dequantized
rotated weights (the codes on their grids).

The oracle is that definition written out: unpack, dequantize, undo BiIP
on the dense matrix, multiply.  (TEST INFRASTRUCTURE ONLY, like the rest
of this package.)
"""

from __future__ import annotations

import numpy as np

from . import biip, pack


def dequantize_layer(codes: np.ndarray, scales: np.ndarray, zeros: np.ndarray, group: int) -> np.ndarray:
    """W_hat'[i, j] = scale[i, g(j)] (code[i, j] - zero[i, g(j)]), fp64;
    g(j) = j // group (0 for per-channel)."""
    codes = np.asarray(codes, dtype=np.float64)
    m, n = codes.shape
    g = n if group == -1 else group
    gi = np.arange(n) // g
    s = np.asarray(scales, dtype=np.float64)[:, gi]
    z = np.asarray(zeros, dtype=np.float64)[:, gi]
    return s * (codes - z)


def deploy_weights(packed, n, bits, group, scales, zeros, S_X, S_G, sign_u, sign_v, mode="full"):
    """The original-space W_hat the packed layer stands for."""
    codes = pack.unpack(np.asarray(packed), n, bits)
    Whp = dequantize_layer(codes, scales, zeros, group)
    return biip.unbiip_w(Whp, S_X, S_G, sign_u, sign_v, mode)


def deploy_matvec(packed, n, bits, group, scales, zeros, S_X, S_G, sign_u, sign_v, x, mode="full"):
    """y = W_hat x for each row of x (batch x n) -> batch x m."""
    W = deploy_weights(packed, n, bits, group, scales, zeros, S_X, S_G, sign_u, sign_v, mode)
    return np.asarray(x, dtype=np.float64) @ W.T
