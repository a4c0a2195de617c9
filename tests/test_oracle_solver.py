"""Pins of the oracle's grid, inverse Cholesky factor and OBS column loop.

* Proposition 1 (KronQ summary (hyper.ai), "Method"; KronQ review
  (pith.science), appendix A.1): the group-OBS update with the full
  Kronecker Hessian H_X (x) H_G equals the H_X-only column update row by row.
  Checked with an independent route: explicit inverse of the mn x mn
  Hessian, column-group OBS step and inverse downdate.
* Exhaustive search over all codes on tiny rows: the OBS loop's loss is
  never below the optimum, equals it for one column, and beats
  round-to-nearest in most trials.
* Closed forms: two columns; diagonal H; one column; U^T U H = I.
* Exact bookkeeping: dW_i H dW_i^T = sum_j e_ij^2 for every row.
"""

import itertools

import numpy as np
import pytest

from conftest import GOLDEN
from oracle import cholesky as C
from oracle import quantizer as Q


def _spd(r, d, cond=50.0):
    A = r.standard_normal((d, d))
    Qm, _ = np.linalg.qr(A)
    ev = np.exp(np.linspace(0, np.log(cond), d))
    return (Qm * ev) @ Qm.T


# ----------------------------------------------------------------- grid
def test_grid_golden_2bit():
    line = (GOLDEN / "grid_2bit.txt").read_text().splitlines()[-1]
    w, zero, q, wh = [np.array(p.split(), dtype=float) for p in line.split("|")]
    scale, z = Q.grid_params(w, 2)
    assert z[0] == int(zero[0])
    np.testing.assert_allclose(scale[0], 4.0 / 3.0, rtol=1e-7)
    codes = Q.quantize(w, scale[0], z[0], 2)
    np.testing.assert_array_equal(codes, q.astype(int))
    np.testing.assert_allclose(Q.dequantize(codes, scale[0], z[0]), wh, rtol=1e-6)


def test_grid_zero_row_and_ties():
    s, z = Q.grid_params(np.zeros((2, 5)), 4)
    assert np.all(s == 1) and np.all(z == 0)
    # ties go to even: 0.5 -> 0, 1.5 -> 2, 2.5 -> 2
    q = Q.quantize(np.array([0.5, 1.5, 2.5]), np.float32(1.0), 0, 4)
    np.testing.assert_array_equal(q, [0, 2, 2])
    # clamping at both ends
    q = Q.quantize(np.array([-9.0, 99.0]), np.float32(1.0), 3, 2)
    np.testing.assert_array_equal(q, [0, 3])


def test_grid_all_positive_and_all_negative():
    s, z = Q.grid_params(np.array([[0.5, 1.0, 3.0]]), 2)
    assert z[0] == 0                          # lo clamps to 0
    s, z = Q.grid_params(np.array([[-0.5, -1.0, -3.0]]), 2)
    assert z[0] == 3                          # hi clamps to 0
    q = Q.quantize(np.array([-3.0, 0.0]), s[0], z[0], 2)
    np.testing.assert_array_equal(q, [0, 3])


# ------------------------------------------------------ inverse Cholesky
def test_inverse_cholesky_definition():
    r = np.random.default_rng(1)
    H = _spd(r, 30, cond=1e3)
    U = C.inverse_cholesky(H)
    assert np.allclose(np.tril(U, -1), 0)
    assert np.all(np.diag(U) > 0)
    np.testing.assert_allclose(U.T @ U @ H, np.eye(30), atol=1e-10)


def test_inverse_cholesky_diagonal_closed_form():
    h = np.array([4.0, 9.0, 0.25, 1.0])
    np.testing.assert_allclose(C.inverse_cholesky(np.diag(h)), np.diag(h ** -0.5), rtol=1e-15)


def test_inverse_cholesky_2x2_closed_form():
    a, b, c = 4.0, 2.0, 3.0
    U = C.inverse_cholesky(np.array([[a, b], [b, c]]))
    det = a * c - b * b
    np.testing.assert_allclose(U[0, 0], np.sqrt(c / det), rtol=1e-14)
    np.testing.assert_allclose(U[0, 1] / U[0, 0], -b / c, rtol=1e-14)
    np.testing.assert_allclose(U[1, 1], 1 / np.sqrt(c), rtol=1e-14)


def test_damp_and_not_pd():
    H = np.array([[2.0, 0.0], [0.0, 4.0]])
    np.testing.assert_allclose(C.damp(H, 0.01), H + 0.03 * np.eye(2))
    with pytest.raises(C.NotPositiveDefinite):
        C.inverse_cholesky(np.array([[1.0, 2.0], [2.0, 1.0]]))


# ------------------------------------------------------------ the solver
def test_two_column_closed_form_golden():
    line = (GOLDEN / "gptq_2col.txt").read_text().splitlines()[-1]
    f = [np.array(p.split(), dtype=float) for p in line.split("|")]
    H = f[0].reshape(2, 2)
    w, bits, q, wh, w2u = f[1], int(f[2][0]), f[3], f[4], f[5][0]
    res = Q.obs_quantize(w[None, :], C.inverse_cholesky(H), bits, -1)
    np.testing.assert_array_equal(res["codes"][0], q.astype(int))
    np.testing.assert_allclose(res["W_hat"][0], wh, rtol=1e-6)
    # the compensated second weight: quantized value + scaled error * U[1, 1]
    U = C.inverse_cholesky(H)
    np.testing.assert_allclose(res["W_hat"][0, 1] + res["E"][0, 1] * U[1, 1], w2u, rtol=1e-6)


def _kron_obs(W, HX, HG, bits):
    """Independent route: sequential group OBS with the full Kronecker Hessian.
    vec is column-stacking (index j*m + i for W[i, j])."""
    m, n = W.shape
    Hfull = np.kron(HX, HG)
    Hinv = np.linalg.inv(Hfull)
    w = W.reshape(-1, order="F").copy()
    scale, zero = Q.grid_params(W, bits)
    alive = list(range(m * n))
    codes = np.zeros((m, n), dtype=int)
    for p in range(n):
        P = [p * m + i for i in range(m)]
        R = [k for k in alive if k not in P]
        q = Q.quantize(w[P], scale, zero, bits)
        codes[:, p] = q
        delta = w[P] - Q.dequantize(q, scale, zero)
        ia = [alive.index(k) for k in P]
        ir = [alive.index(k) for k in R]
        Hpp = Hinv[np.ix_(ia, ia)]
        Hrp = Hinv[np.ix_(ir, ia)]
        sol = np.linalg.solve(Hpp, delta)
        w[R] -= Hrp @ sol
        w[P] = Q.dequantize(q, scale, zero)
        Hinv = Hinv[np.ix_(ir, ir)] - Hrp @ np.linalg.solve(Hpp, Hrp.T)
        alive = R
    return codes, w.reshape((m, n), order="F")


@pytest.mark.parametrize("m,n,bits", [(4, 6, 2), (3, 8, 4), (6, 5, 3)])
def test_proposition1_kronecker_obs_equals_column_loop(m, n, bits):
    r = np.random.default_rng(m * 10 + n)
    W = r.standard_normal((m, n))
    HX = C.damp(_spd(r, n, cond=30.0), 0.01)
    HG = _spd(r, m, cond=1e3)                      # strongly non-identity H_G
    codes_k, what_k = _kron_obs(W, HX, HG, bits)
    res = Q.obs_quantize(W, C.inverse_cholesky(HX), bits, -1)
    np.testing.assert_array_equal(res["codes"], codes_k)
    np.testing.assert_allclose(res["W_hat"], what_k, atol=1e-9)


def test_per_row_error_identity():
    r = np.random.default_rng(5)
    m, n = 7, 40
    W = r.standard_normal((m, n))
    H = C.damp(_spd(r, n, cond=200.0), 0.01)
    res = Q.obs_quantize(W, C.inverse_cholesky(H), 3, -1)
    lhs = Q.row_losses(W - res["W_hat"], H)
    rhs = (res["E"] ** 2).sum(axis=1)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-9)


def test_group_mode_identity_and_params():
    r = np.random.default_rng(6)
    m, n, g = 5, 32, 8
    W = r.standard_normal((m, n))
    H = C.damp(_spd(r, n, cond=100.0), 0.01)
    res = Q.obs_quantize(W, C.inverse_cholesky(H), 2, g)
    assert res["scale"].shape == (m, n // g)
    np.testing.assert_allclose(Q.row_losses(W - res["W_hat"], H), (res["E"] ** 2).sum(1), rtol=1e-9)
    # every W_hat value sits on its group's grid
    for b in range(n // g):
        sl = slice(b * g, (b + 1) * g)
        k = (res["W_hat"][:, sl] / res["scale"][:, b:b + 1].astype(float)) + res["zero"][:, b:b + 1]
        np.testing.assert_allclose(k, res["codes"][:, sl], atol=1e-5)


def _exhaustive(w, H, scale, zero, bits):
    maxq = 2 ** bits - 1
    best = np.inf
    for q in itertools.product(range(maxq + 1), repeat=len(w)):
        d = w - Q.dequantize(np.array(q), scale, zero)
        best = min(best, float(d @ H @ d))
    return best


@pytest.mark.parametrize("n,bits", [(6, 2), (4, 4), (1, 2), (1, 4)])
def test_exhaustive_optimum_bounds_obs(n, bits):
    r = np.random.default_rng(100 + n * bits)
    wins = 0
    trials = 12
    for t in range(trials):
        w = r.standard_normal(n)
        H = C.damp(_spd(r, n, cond=80.0), 0.01)
        res = Q.obs_quantize(w[None, :], C.inverse_cholesky(H), bits, -1)
        rtn = Q.rtn_quantize(w[None, :], bits, -1)
        scale, zero = res["scale"][0, 0], int(res["zero"][0, 0])
        l_obs = float(Q.row_losses(w[None, :] - res["W_hat"], H)[0])
        l_rtn = float(Q.row_losses(w[None, :] - rtn["W_hat"], H)[0])
        l_opt = _exhaustive(w, H, scale, zero, bits)
        assert l_opt <= l_obs * (1 + 1e-12) + 1e-15
        if n == 1:
            assert abs(l_obs - l_opt) <= 1e-12 * max(1.0, l_opt)
            assert abs(l_rtn - l_opt) <= 1e-12 * max(1.0, l_opt)
        wins += l_obs <= l_rtn * (1 + 1e-12)
    assert wins >= trials * 2 // 3


def test_diagonal_hessian_reduces_to_rtn():
    r = np.random.default_rng(9)
    W = r.standard_normal((6, 16))
    H = np.diag(r.uniform(0.5, 5.0, 16))
    res = Q.obs_quantize(W, C.inverse_cholesky(H), 3, -1)
    rtn = Q.rtn_quantize(W, 3, -1)
    np.testing.assert_array_equal(res["codes"], rtn["codes"])


def test_obs_rows_subset_matches_full():
    r = np.random.default_rng(10)
    W = r.standard_normal((130, 24))
    U = C.inverse_cholesky(C.damp(_spd(r, 24), 0.01))
    full = Q.obs_quantize(W, U, 4, -1)
    rows = np.array([0, 3, 64, 65, 129])
    sub = Q.obs_quantize_rows(W, U, 4, -1, rows=rows, chunk=2, threads=3)
    np.testing.assert_array_equal(sub["codes"], full["codes"][rows])
    np.testing.assert_array_equal(sub["W_hat"], full["W_hat"][rows])


def test_bad_arguments():
    with pytest.raises(ValueError):
        Q.obs_quantize(np.zeros((2, 10)), np.eye(10), 4, 3)
    with pytest.raises(ValueError):
        Q.obs_quantize(np.zeros((2, 10)), np.eye(10), 5, -1)


def test_layer_loss_matches_kronecker_quadratic_form():
    r = np.random.default_rng(12)
    m, n = 3, 4
    dW = r.standard_normal((m, n))
    HX, HG = _spd(r, n), _spd(r, m)
    v = dW.reshape(-1, order="F")
    np.testing.assert_allclose(Q.layer_loss(dW, HX, HG), v @ np.kron(HX, HG) @ v, rtol=1e-12)


@pytest.mark.parametrize("n,k", [(40, 0), (40, 17), (64, 63), (100, 36)])
def test_inverse_cholesky_trailing_block(n, k):
    """U[k:, k:] depends on H[k:, k:] only (upper factor of the inverse)."""
    r = np.random.default_rng(n + k)
    H = _spd(r, n)
    np.testing.assert_allclose(C.inverse_cholesky_trailing(H, k, 0.01),
                               C.inverse_cholesky(C.damp(H, 0.01))[k:, k:], rtol=1e-9, atol=1e-12)


def test_row_losses_damping_argument_and_fp32_input():
    r = np.random.default_rng(21)
    n = 2100                                   # more than one 2048-row panel
    H = _spd(r, n)
    dW = r.standard_normal((3, n))
    ref = np.einsum("ij,jk,ik->i", dW, C.damp(H, 0.01), dW)
    np.testing.assert_allclose(Q.row_losses(dW, H, 0.01), ref, rtol=1e-11)
    H32 = H.astype(np.float32)
    np.testing.assert_allclose(Q.row_losses(dW, H32), np.einsum("ij,jk,ik->i", dW, H32.astype(np.float64), dW),
                               rtol=1e-11)


def test_ldlq_quarter_bound_table9():
    """KronQ review (pith.science), reference-list fragment of the appendix,
    Table 9 (worst-case proxy loss under LDLQ rounding, GPTQ-LDLQ with
    H_G = I): with rounding errors of at most half a grid step, a row's loss
    under the column loop is at most 1/4 step^2 tr(D_X), D_X the diagonal of
    the LDL factorisation of H in the loop's order.  D_X is taken here from a
    Cholesky factor of the index-reversed H (not from the oracle's factor):
    it must equal 1 / U[j, j]^2, and the loop's loss sum_j e_j^2 must respect
    the bound on every row whose rounding errors stayed within half a step
    (a value pushed past the grid's end is clamped and may err by more)."""
    r = np.random.default_rng(41)
    m, n, bits = 24, 64, 8
    W = r.standard_normal((m, n))
    Hd = C.damp(_spd(r, n, cond=200.0), 0.01)
    U = C.inverse_cholesky(Hd)
    Lr = np.linalg.cholesky(Hd[::-1, ::-1])
    D = (np.diag(Lr) ** 2)[::-1]
    np.testing.assert_allclose(1.0 / np.diag(U) ** 2, D, rtol=1e-9)
    res = Q.obs_quantize(W, U, bits)
    checked = 0
    for i in range(m):
        step = float(res["scale"][i, 0])
        rerr = res["E"][i] * np.diag(U)              # w_j - w_hat_j at quantization time
        if np.max(np.abs(rerr)) > 0.5 * step * (1 + 1e-6):
            continue
        assert np.sum(res["E"][i] ** 2) <= 0.25 * step ** 2 * np.sum(D) * (1 + 1e-9)
        checked += 1
    assert checked >= m // 2, checked


@pytest.mark.parametrize("m,n,bits,group", [(37, 256, 4, -1), (20, 384, 2, 128), (9, 128, 3, 32),
                                            (17, 512, 2, 64), (1, 128, 4, 128), (0, 128, 4, -1)])
def test_c_loop_is_bit_identical_to_the_numpy_loop(m, n, bits, group):
    """oracle/c/obs_rows.c restates obs_quantize in C for wide layers: the
    same fp32 decisions and fp64 updates in the same order, so every code,
    grid and W_hat entry must agree bit for bit, on rows with outliers and
    an all-zero row too."""
    from oracle import cholesky as ochol
    r = np.random.default_rng(m * 7 + n)
    A = r.standard_normal((2 * n, n)) * np.exp(r.uniform(-1, 1, n))
    U = ochol.inverse_cholesky(ochol.damp(A.T @ A / (2 * n), 0.01))
    W = r.standard_normal((m, n)) * 0.02
    if m > 2:
        W[1] = 0.0
        W[2, :: max(1, n // 5)] *= 40.0
    a = Q.obs_quantize(W, U, bits, group)
    rows = np.arange(m)[::-1].copy()
    b = Q.obs_quantize_rows_c(W, U, bits, group, rows=rows)
    for k in ("codes", "scale", "zero", "W_hat"):
        assert np.array_equal(a[k][rows], b[k]), k
