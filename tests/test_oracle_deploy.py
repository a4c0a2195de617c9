"""Pins of the oracle's deployment matvec (oracle/deploy.py).

* The BiIP undo on the deploy path against the dense transform matrices:
  W = S_G^-1 (T_m D_u)^T W' (T_n D_v) S_X^-1 built from explicit matrices
  (not the fast transform the oracle uses), for every --incoh_mode.
* The output error of the deployed layer against the loss the solver sees:
  sum_t ||W_hat x_t - W x_t||^2 / N = tr(H_G' dW' H_X' dW'^T) with
  H_X = X^T X / N, H_G = I, computed in the rotated space (Thm 1 carries it
  over; KronQ review (pith.science), appendix A.2).
* Dequantization on a hand-worked row.
"""

import numpy as np
import pytest

from oracle import biip, deploy, pack, quantizer, transform


def _layer(r, m, n, bits, group):
    G = 1 if group == -1 else n // group
    codes = r.integers(0, 2 ** bits, (m, n)).astype(np.uint8)
    scales = r.uniform(0.01, 0.05, (m, G)).astype(np.float32)
    zeros = r.integers(0, 2 ** bits, (m, G)).astype(np.uint8)
    return codes, scales, zeros


def test_dequantize_hand_worked():
    codes = np.array([[0, 1, 2, 3, 3, 2, 1, 0]], dtype=np.uint8)
    scales = np.array([[0.5, 2.0]], dtype=np.float32)
    zeros = np.array([[1, 2]], dtype=np.uint8)
    W = deploy.dequantize_layer(codes, scales, zeros, 4)
    np.testing.assert_array_equal(W, [[-0.5, 0.0, 0.5, 1.0, 2.0, 0.0, -2.0, -4.0]])


@pytest.mark.parametrize("mode", biip.MODES)
@pytest.mark.parametrize("m,n,bits,group", [(64, 48, 4, -1), (96, 64, 2, 32), (112, 128, 4, 64)])
def test_unrotation_against_dense_transforms(mode, m, n, bits, group):
    r = np.random.default_rng(m + n + bits)
    codes, scales, zeros = _layer(r, m, n, bits, group)
    su = (1 - 2 * r.integers(0, 2, m)).astype(np.int8)
    sv = (1 - 2 * r.integers(0, 2, n)).astype(np.int8)
    in_s, out_s, in_r, out_r = biip.sides(mode)
    SX = r.uniform(0.5, 2.0, n) if in_s else np.ones(n)
    SG = r.uniform(0.5, 2.0, m) if out_s else np.ones(m)
    x = r.standard_normal((3, n))
    Wq = deploy.dequantize_layer(codes, scales, zeros, group)
    U = transform.dense(m, su) if out_r else np.eye(m)
    V = transform.dense(n, sv) if in_r else np.eye(n)
    W = np.diag(1 / SG) @ U.T @ Wq @ V @ np.diag(1 / SX)
    y = deploy.deploy_matvec(pack.pack(codes, bits), n, bits, group, scales, zeros, SX, SG, su, sv,
                             x, mode)
    np.testing.assert_allclose(y, x @ W.T, rtol=1e-10, atol=1e-12)


def test_output_error_equals_rotated_space_loss():
    r = np.random.default_rng(5)
    m, n, N = 32, 64, 4000
    W = r.standard_normal((m, n)) * 0.02
    X = r.standard_normal((N, n)) * np.exp(r.uniform(-1, 1, n))
    HX = X.T @ X / N
    HG = np.eye(m)
    su = (1 - 2 * r.integers(0, 2, m)).astype(np.int8)
    sv = (1 - 2 * r.integers(0, 2, n)).astype(np.int8)
    Wp, HXt, HGt, SX, SG = biip.biip(W, HX, HG, su, sv, 0.25, "full")
    res = quantizer.rtn_quantize(Wp, 4)
    y = deploy.deploy_matvec(pack.pack(res["codes"], 4), n, 4, -1, res["scale"], res["zero"], SX, SG,
                             su, sv, X)
    out_err = np.sum((y - X @ W.T) ** 2) / N
    loss_rot = quantizer.layer_loss(Wp - res["W_hat"], HXt, HGt)
    np.testing.assert_allclose(out_err, loss_rot, rtol=1e-9)
