"""Asymmetric b-bit grid, the column-wise OBS solver and the layer loss.

Sources:
  * KronQ summary (hyper.ai), "Method": the Kronecker-factored objective
    tr(H_G dW H_X dW^T), dW = W - W_hat; under the column-wise OBS update the
    compensation after quantizing column p uses only H_X's inverse factor,
    H_G cancels (Proposition 1).
  * KronQ review (pith.science), appendix, Algorithm 2: damping, inverse
    Cholesky, then a loop over columns in blocks of B with an error buffer E.
    Blocking is a reassociation of the same column loop; the oracle runs the
    plain unblocked loop: after column j, every later column k is updated at
    once.
  * KronQ README (GitHub), "Reproduce from scratch": --w_asym, --w_groupsize
    -1 (per-channel) or 128, 2/3/4 bits, and the flags --w_clip and
    --act_order, which the pages name but do not define (readings below;
    both are off unless asked for).

Readings:
  * grid: lo = min(0, min w), hi = max(0, max w), scale = (hi - lo)/(2^b - 1),
    zero = round(-lo / scale); a row or group that is all zero gets
    scale = 1, zero = 0.
  * code: q = clamp(round(w / scale) + zero, 0, 2^b - 1), w_hat = scale (q - zero);
    round = half to even.
  * The decisions that produce integers (scale, zero, q) are taken in fp32,
    the precision the CUDA kernels take them in: w is cast to fp32, then the
    fp32 operations above are applied in that order.
  * per-channel parameters come from the whole row of W' before the loop;
    group parameters at column j = 0 mod g from the current (already
    error-updated) columns j .. j+g-1.
  * column update: e = (w_j - w_hat_j) / U[j, j]; W[:, k] -= e U[j, k], k > j.
  * --w_clip (reading): for each row (per-channel) or group, the grid is
    chosen among the shrunk ranges [p lo, p hi], p = 1 - i/100 for
    i = 0 .. 79, as the first one with the smallest squared quantization
    error sum_k (w_k - w_hat_k)^2 over the row or group.  The grid of each
    candidate and the differences w_k - w_hat_k are fp32 operations (the
    decision precision above); the squares of those fp32 differences are
    exact in fp64 and are summed in fp64, so that the choice does not hinge
    on the order of the sum.
  * --act_order (reading): act_order_perm below.
"""

from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np

F32 = np.float32


def grid_params(w: np.ndarray, bits: int):
    """Per-row (scale fp32, zero int) of the asymmetric grid for each row of w."""
    w32 = np.asarray(w, dtype=np.float64).astype(F32)
    if w32.ndim == 1:
        w32 = w32[None, :]
    maxq = F32(2 ** bits - 1)
    lo = np.minimum(w32.min(axis=1), F32(0))
    hi = np.maximum(w32.max(axis=1), F32(0))
    zero_row = (lo == 0) & (hi == 0)
    span = (hi - lo).astype(F32)
    span[zero_row] = maxq
    scale = (span / maxq).astype(F32)
    zero = np.rint((-lo).astype(F32) / scale).astype(F32)
    zero = np.clip(zero, F32(0), maxq)
    scale[zero_row] = F32(1)
    zero[zero_row] = F32(0)
    return scale, zero.astype(np.int64)


CLIP_GRID = 100      # candidate shrink ratios p = 1 - i / CLIP_GRID ...
CLIP_STEPS = 80      # ... for i = 0 .. CLIP_STEPS - 1


def clip_ratio(i: int) -> np.float32:
    """p_i = 1 - i/100, evaluated in fp64 and rounded once to fp32."""
    return F32(1.0 - i * (1.0 / CLIP_GRID))


def _grid_from_range(lo: np.ndarray, hi: np.ndarray, bits: int):
    """(scale, zero) of the asymmetric grid of [lo, hi] (fp32, lo <= 0 <= hi)."""
    maxq = F32(2 ** bits - 1)
    zero_row = (lo == 0) & (hi == 0)
    span = (hi - lo).astype(F32)
    span[zero_row] = maxq
    scale = (span / maxq).astype(F32)
    zero = np.rint((-lo).astype(F32) / scale).astype(F32)
    zero = np.clip(zero, F32(0), maxq)
    scale[zero_row] = F32(1)
    zero[zero_row] = F32(0)
    return scale, zero.astype(np.int64)


def sq_error(w32: np.ndarray, scale, zero, bits: int) -> np.ndarray:
    """Per-row sum of (w - w_hat)^2: w_hat = scale (q - zero) and the
    difference in fp32, the squares (exact) and their sum in fp64."""
    scale = np.asarray(scale, dtype=F32).reshape(-1, 1)
    zero = np.asarray(zero, dtype=np.int64).reshape(-1, 1)
    q = quantize(w32, scale, zero, bits)
    wh = (scale * (q - zero).astype(F32)).astype(F32)
    d = (w32 - wh).astype(F32).astype(np.float64)
    return np.sum(d * d, axis=1)


def clip_grid_params(w: np.ndarray, bits: int):
    """Per-row (scale, zero) of the --w_clip search (reading in the module
    docstring): the first of the shrunk grids with the least squared error."""
    w32 = np.asarray(w, dtype=np.float64).astype(F32)
    if w32.ndim == 1:
        w32 = w32[None, :]
    lo = np.minimum(w32.min(axis=1), F32(0))
    hi = np.maximum(w32.max(axis=1), F32(0))
    best = np.full(w32.shape[0], np.inf)
    scale = np.ones(w32.shape[0], dtype=F32)
    zero = np.zeros(w32.shape[0], dtype=np.int64)
    for i in range(CLIP_STEPS):
        p = clip_ratio(i)
        s1, z1 = _grid_from_range((lo * p).astype(F32), (hi * p).astype(F32), bits)
        err = sq_error(w32, s1, z1, bits)
        better = err < best
        best[better] = err[better]
        scale[better] = s1[better]
        zero[better] = z1[better]
    return scale, zero


def quantize(w: np.ndarray, scale: np.ndarray, zero: np.ndarray, bits: int) -> np.ndarray:
    """Integer codes, decided in fp32 (reading in the module docstring)."""
    maxq = 2 ** bits - 1
    w32 = np.asarray(w, dtype=np.float64).astype(F32)
    r = np.rint(w32 / np.asarray(scale, dtype=F32)).astype(np.int64)
    return np.clip(r + np.asarray(zero, dtype=np.int64), 0, maxq)


def dequantize(q, scale, zero) -> np.ndarray:
    return np.asarray(scale, dtype=np.float64) * (np.asarray(q, dtype=np.int64)
                                                 - np.asarray(zero, dtype=np.int64))


def _check(n: int, group: int, bits: int):
    if bits not in (2, 3, 4, 8):
        raise ValueError("bits must be 2, 3, 4 or 8")
    if group != -1 and (group <= 0 or n % group):
        raise ValueError("group must be -1 or divide n")


def obs_quantize(W: np.ndarray, U: np.ndarray, bits: int, group: int = -1, clip: bool = False):
    """Unblocked column-wise OBS loop on the rows of W (rows are independent).

    W: m x n (the rotated weights, widened to fp64).  U: n x n upper inverse
    Cholesky factor of the damped H_X.  clip: the --w_clip grid search.
    Returns a dict with codes (m x n), scale and zero (m x n_groups), W_hat
    (m x n) and the scaled errors E."""
    params = clip_grid_params if clip else grid_params
    W = np.array(W, dtype=np.float64)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    _check(n, group, bits)
    ng = 1 if group == -1 else n // group
    codes = np.zeros((m, n), dtype=np.uint8)
    scales = np.zeros((m, ng), dtype=F32)
    zeros = np.zeros((m, ng), dtype=np.uint8)
    What = np.zeros((m, n))
    E = np.zeros((m, n))
    if group == -1:
        scale, zero = params(W, bits)
        scales[:, 0], zeros[:, 0] = scale, zero
    for j in range(n):
        if group != -1 and j % group == 0:
            scale, zero = params(W[:, j:j + group], bits)
            scales[:, j // group], zeros[:, j // group] = scale, zero
        w = W[:, j]
        q = quantize(w, scale, zero, bits)
        wh = dequantize(q, scale, zero)
        e = (w - wh) / U[j, j]
        W[:, j + 1:] -= np.outer(e, U[j, j + 1:])
        codes[:, j] = q
        What[:, j] = wh
        E[:, j] = e
    return {"codes": codes, "scale": scales, "zero": zeros, "W_hat": What, "E": E}


def obs_quantize_rows(W: np.ndarray, U: np.ndarray, bits: int, group: int = -1,
                      rows=None, chunk: int = 64, threads: int | None = None, clip: bool = False):
    """obs_quantize on a subset of rows, in row chunks on a thread pool.

    Each row's arithmetic is exactly that of obs_quantize: the rows of the
    loop never interact, so splitting them changes no operation."""
    W = np.asarray(W)
    rows = np.arange(W.shape[0]) if rows is None else np.asarray(rows)
    parts = [rows[i:i + chunk] for i in range(0, len(rows), chunk)]
    threads = threads or min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(threads) as ex:
        res = list(ex.map(lambda r: obs_quantize(W[r], U, bits, group, clip), parts))
    if not res:
        return obs_quantize(W[:0], U, bits, group, clip)
    return {k: np.concatenate([r[k] for r in res], axis=0) for k in res[0]}


def obs_quantize_rows_c(W: np.ndarray, U: np.ndarray, bits: int, group: int = -1, rows=None,
                        threads: int | None = None):
    """obs_quantize on a subset of rows through the plain-C restatement of
    the same loop (oracle/c/obs_rows.c: the same fp32 decisions and fp64
    updates in the same order, without floating-point contraction), for
    wide layers where the numpy loop is too slow.  Results are bit-identical
    to obs_quantize (pinned in the oracle tests).  No --w_clip here."""
    import ctypes
    from . import build_c
    lib = ctypes.CDLL(str(build_c.build()))
    f = lib.kronq_oracle_obs_rows
    P = ctypes.c_void_p
    f.argtypes = [P, ctypes.c_int64, ctypes.c_int64, P, ctypes.c_int, ctypes.c_int, P, P, P, P,
                  ctypes.c_int]
    f.restype = ctypes.c_int
    W = np.asarray(W)
    rows = np.arange(W.shape[0]) if rows is None else np.asarray(rows)
    n = W.shape[1]
    _check(n, group, bits)
    Wr = np.ascontiguousarray(W[rows], dtype=np.float64)
    U = np.ascontiguousarray(U, dtype=np.float64)
    m = Wr.shape[0]
    ng = 1 if group == -1 else n // group
    codes = np.zeros((m, n), dtype=np.uint8)
    scales = np.zeros((m, ng), dtype=F32)
    zeros = np.zeros((m, ng), dtype=np.uint8)
    What = np.zeros((m, n))
    if m:
        st = f(Wr.ctypes.data, m, n, U.ctypes.data, bits, group, codes.ctypes.data,
               scales.ctypes.data, zeros.ctypes.data, What.ctypes.data,
               int(threads or (os.cpu_count() or 1)))
        if st != 0:
            raise ValueError("oracle C loop rejected its arguments")
    return {"codes": codes, "scale": scales, "zero": zeros, "W_hat": What}


def act_order_perm(H: np.ndarray) -> np.ndarray:
    """--act_order (reading): the columns are quantized in descending order
    of the diagonal of the (rotated, undamped) H_X handed to the solver, equal
    diagonals in increasing column order.  perm[k] = the column quantized
    k-th.  The solver then runs on W[:, perm] with H[perm][:, perm] (damping
    and inverse Cholesky of the permuted matrix), and its codes and W_hat go
    back to the original column order; with groups, a group is g consecutive
    columns of the permuted order."""
    d = np.asarray(np.diag(np.asarray(H)), dtype=np.float64)
    return np.array(sorted(range(len(d)), key=lambda j: (-d[j], j)), dtype=np.int64)


def obs_quantize_act_order(W: np.ndarray, H_damped: np.ndarray, perm: np.ndarray, bits: int,
                           group: int = -1, clip: bool = False, rows=None):
    """The column loop in the order perm (act_order_perm), results in the
    original column order.  H_damped: the damped H_X (unpermuted); its
    permuted copy gets its own inverse Cholesky factor.  scale / zero are
    indexed by groups of the permuted order."""
    from . import cholesky
    perm = np.asarray(perm)
    Up = cholesky.inverse_cholesky(np.asarray(H_damped, dtype=np.float64)[np.ix_(perm, perm)])
    Wp = np.asarray(W, dtype=np.float64)[:, perm]
    res = obs_quantize_rows(Wp, Up, bits, group, rows=rows, clip=clip)
    out = dict(res)
    for k in ("codes", "W_hat", "E"):
        back = np.empty_like(res[k])
        back[:, perm] = res[k]
        out[k] = back
    out["U_perm"] = Up
    return out


def rtn_quantize(W: np.ndarray, bits: int, group: int = -1):
    """Round-to-nearest on the same grid (no error propagation)."""
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    _check(n, group, bits)
    g = n if group == -1 else group
    codes = np.zeros((m, n), dtype=np.uint8)
    What = np.zeros((m, n))
    scales = np.zeros((m, n // g), dtype=F32)
    zeros = np.zeros((m, n // g), dtype=np.uint8)
    for b in range(n // g):
        sl = slice(b * g, (b + 1) * g)
        scale, zero = grid_params(W[:, sl], bits)
        q = quantize(W[:, sl], scale[:, None], zero[:, None], bits)
        codes[:, sl] = q
        What[:, sl] = dequantize(q, scale[:, None], zero[:, None])
        scales[:, b], zeros[:, b] = scale, zero
    return {"codes": codes, "scale": scales, "zero": zeros, "W_hat": What}


def layer_loss(dW: np.ndarray, HX: np.ndarray, HG: np.ndarray) -> float:
    """tr(H_G dW H_X dW^T), fp64."""
    dW = np.asarray(dW, dtype=np.float64)
    M = np.asarray(HG, dtype=np.float64) @ dW @ np.asarray(HX, dtype=np.float64)
    return float(np.sum(M * dW))


def row_losses(dW: np.ndarray, HX: np.ndarray, lam: float = 0.0) -> np.ndarray:
    """dW_i H dW_i^T for each row (the part of the loss the solver sees),
    with H = H_X + lam * mean(diag(H_X)) I (lam = 0: H_X itself).  H_X may be
    fp32; it is widened to fp64 one row panel at a time."""
    dW = np.asarray(dW, dtype=np.float64)
    n = dW.shape[1]
    P = np.zeros_like(dW)
    for p in range(0, n, 2048):
        P += dW[:, p:p + 2048] @ np.asarray(HX[p:p + 2048], dtype=np.float64)
    out = np.einsum("ij,ij->i", P, dW)
    if lam:
        mu = float(np.mean(np.diag(HX).astype(np.float64)))
        out += lam * mu * np.einsum("ij,ij->i", dW, dW)
    return out
