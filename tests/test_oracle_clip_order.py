"""Pins of the oracle's --w_clip grid search and --act_order column order
(KronQ README (GitHub), "Reproduce from scratch": both flags are part of the
base recipe; the pages do not define them, the readings are in
oracle/quantizer.py).

* w_clip: with a single candidate it is the plain min/max grid; a row that
  lies exactly on its full-range grid keeps that grid (zero error); a
  hand-worked outlier row where shrinking wins; the choice equals a
  scalar brute-force search (first minimum) on random rows.
* act_order: the permutation on closed cases (sorted, reversed, ties); on a
  diagonal H_X the OBS loop reduces to round-to-nearest in any column order;
  the permuted loop equals the plain loop run on explicitly permuted inputs,
  mapped back.
"""

import itertools

import numpy as np
import pytest

from oracle import cholesky as C
from oracle import quantizer as Q

F32 = np.float32


# ---------------------------------------------------------------- w_clip
def test_single_candidate_is_the_plain_grid(monkeypatch):
    r = np.random.default_rng(0)
    w = r.standard_normal((20, 48))
    monkeypatch.setattr(Q, "CLIP_STEPS", 1)
    for bits in (2, 3, 4):
        s1, z1 = Q.clip_grid_params(w, bits)
        s0, z0 = Q.grid_params(w, bits)
        np.testing.assert_array_equal(s1, s0)
        np.testing.assert_array_equal(z1, z0)


def test_row_on_its_full_grid_keeps_it():
    # 2-bit grid scale 0.5, zero 1: values -0.5, 0, 0.5, 1.0 with both ends present
    w = np.array([[-0.5, 0.0, 0.5, 1.0, 0.5, -0.5, 1.0, 0.0]])
    s, z = Q.clip_grid_params(w, 2)
    assert s[0] == F32(0.5) and z[0] == 1
    assert Q.sq_error(w.astype(F32), s, z, 2)[0] == 0.0


def test_outlier_row_hand_worked():
    # ten 1.0 and one 3.2, 2 bits: the full range [0, 3.2] has scale 3.2/3,
    # every 1.0 lands on code 1 (1/1.0667 = 0.9375 rounds to 1), i.e. on
    # 1.0666667, error 10 * (0.0666667)^2 = 0.0444444; the outlier is exact.
    w = np.array([[1.0] * 10 + [3.2]])
    s_full, z_full = Q.grid_params(w, 2)
    e_full = Q.sq_error(w.astype(F32), s_full, z_full, 2)[0]
    assert abs(e_full - 10 * (3.2 / 3 - 1.0) ** 2) < 1e-6
    s, z = Q.clip_grid_params(w, 2)
    e = Q.sq_error(w.astype(F32), s, z, 2)[0]
    assert e < e_full and s[0] < s_full[0]
    # e.g. p = 0.94: scale 1.00267, the ones err by 0.00267, the outlier (code 3)
    # by 0.192: 10 * 0.00267^2 + 0.192^2 = 0.0369 < 0.0444
    assert e <= 0.0370


def _brute_clip(row, bits):
    """Scalar search: fp32 grid and differences, exact squares, fp64 sum."""
    maxq = F32(2 ** bits - 1)
    lo0 = min(F32(0), min(F32(v) for v in row))
    hi0 = max(F32(0), max(F32(v) for v in row))
    best, best_sz = None, None
    for i in range(80):
        p = F32(1.0 - i / 100.0)
        lo, hi = F32(lo0 * p), F32(hi0 * p)
        if lo == 0 and hi == 0:
            s, z = F32(1), 0
        else:
            s = F32(F32(hi - lo) / maxq)
            z = int(min(max(np.rint(F32(-lo) / s), 0), maxq))
        err = 0.0
        for v in row:
            v32 = F32(v)
            q = int(min(max(int(np.rint(v32 / s)) + z, 0), int(maxq)))
            wh = F32(s * F32(q - z))
            dd = float(F32(v32 - wh))
            err += dd * dd
        if best is None or err < best:
            best, best_sz = err, (s, z)
    return best_sz


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_clip_equals_scalar_brute_force(bits):
    r = np.random.default_rng(bits)
    w = r.standard_normal((12, 24)) * np.exp(r.uniform(-2, 1, (12, 1)))
    w[::3, 5] *= 6.0                                     # outliers in some rows
    s, z = Q.clip_grid_params(w, bits)
    for i in range(w.shape[0]):
        bs, bz = _brute_clip(w[i], bits)
        assert s[i] == bs and z[i] == bz, i


def test_clip_in_the_group_loop():
    r = np.random.default_rng(3)
    W = r.standard_normal((6, 64))
    W[:, 7] *= 8.0
    U = C.inverse_cholesky(C.damp(np.eye(64) + 0.3 * np.ones((64, 64)), 0.01))
    res = Q.obs_quantize(W, U, 2, group=32, clip=True)
    base = Q.obs_quantize(W, U, 2, group=32, clip=False)
    # the first group's grid is set from the untouched columns: exactly the search
    s, z = Q.clip_grid_params(W[:, :32], 2)
    np.testing.assert_array_equal(res["scale"][:, 0], s)
    np.testing.assert_array_equal(res["zero"][:, 0], z)
    assert not np.array_equal(res["scale"], base["scale"])


# ------------------------------------------------------------- act_order
def test_perm_closed_cases():
    np.testing.assert_array_equal(Q.act_order_perm(np.diag([5.0, 4.0, 3.0])), [0, 1, 2])
    np.testing.assert_array_equal(Q.act_order_perm(np.diag([1.0, 2.0, 3.0, 4.0])), [3, 2, 1, 0])
    np.testing.assert_array_equal(Q.act_order_perm(np.diag([2.0, 5.0, 2.0, 5.0])), [1, 3, 0, 2])


@pytest.mark.parametrize("group", [-1, 8])
def test_diagonal_hessian_reduces_to_rtn_in_any_order(group):
    # With H diagonal the inverse factor is diagonal: no error propagates and
    # every column is rounded to nearest, whatever the order.
    r = np.random.default_rng(7)
    n = 32
    d = r.uniform(0.5, 3.0, n)
    H = np.diag(d)
    W = r.standard_normal((5, n))
    perm = Q.act_order_perm(H)
    assert not np.array_equal(perm, np.arange(n))
    res = Q.obs_quantize_act_order(W, C.damp(H, 0.01), perm, 3, group)
    rtn = Q.rtn_quantize(W[:, perm], 3, group)
    back = np.empty_like(rtn["codes"])
    back[:, perm] = rtn["codes"]
    np.testing.assert_array_equal(res["codes"], back)
    np.testing.assert_array_equal(res["scale"], rtn["scale"])


def test_permuted_loop_equals_loop_on_permuted_inputs():
    r = np.random.default_rng(9)
    n = 24
    A = r.standard_normal((n, 3 * n))
    H = A @ A.T / (3 * n) + np.diag(r.uniform(0, 4, n))
    Hd = C.damp(H, 0.01)
    W = r.standard_normal((7, n))
    perm = Q.act_order_perm(H)
    res = Q.obs_quantize_act_order(W, Hd, perm, 4, -1, clip=True)
    Up = C.inverse_cholesky(Hd[np.ix_(perm, perm)])
    ref = Q.obs_quantize(W[:, perm], Up, 4, -1, clip=True)
    np.testing.assert_array_equal(res["codes"][:, perm], ref["codes"])
    np.testing.assert_allclose(res["W_hat"][:, perm], ref["W_hat"])
    # the loss bookkeeping of the permuted solve holds in the original order:
    # dW_i Hd dW_i^T = sum_j e_ij^2
    dW = W - res["W_hat"]
    lhs = np.einsum("ij,jk,ik->i", dW, Hd, dW)
    np.testing.assert_allclose(lhs, np.sum(res["E"] ** 2, axis=1), rtol=1e-9)


def test_act_order_never_beats_exhaustive_optimum():
    r = np.random.default_rng(11)
    n, bits = 4, 2
    for _ in range(10):
        A = r.standard_normal((n, 2 * n))
        H = A @ A.T + np.diag(r.uniform(0, 3, n))
        Hd = C.damp(H, 0.01)
        W = r.standard_normal((1, n))
        perm = Q.act_order_perm(H)
        res = Q.obs_quantize_act_order(W, Hd, perm, bits)
        s, z = Q.grid_params(W, bits)
        best = np.inf
        for q in itertools.product(range(2 ** bits), repeat=n):
            dw = W[0] - Q.dequantize(np.array(q), s[0], z[0])
            best = min(best, dw @ Hd @ dw)
        dw = W[0] - res["W_hat"][0]
        assert dw @ Hd @ dw >= best - 1e-12
