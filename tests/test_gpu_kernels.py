"""Parity of every libkronq entry point with the fp64 oracle, through the C
ABI, on seeded inputs sized to span several tiles with ragged tails.

Tolerances (the parity bar): covariances <= 1e-4 relative Frobenius
(bf16 inputs, fp32 accumulation); packing bit-exact; codes >= 99.9 %
identical with the row loss within 1 %.  Rotation and inverse Cholesky are
intermediate fp32 stages: their bound (1e-5 and 1e-4 relative Frobenius)
comes from fp32 rounding over log2(d) butterfly stages and from the
conditioning of the damped matrix.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import bf16_dev, bf16_host, rel_fro, signs, spd, t, widen
from oracle import biip as obiip
from oracle import cholesky as ochol
from oracle import covariance as ocov
from oracle import pack as opack
from oracle import quantizer as oq
from post_quantization_02_b200 import abi

pytestmark = pytest.mark.gpu


def _x(r, N, d, kind="t4"):
    if kind == "t4":
        z = r.standard_normal((N, d)) / np.sqrt(r.gamma(2.0, size=(N, d)) / 2.0)
        z[:, r.permutation(d)[: max(1, d // 200)]] *= 20.0
    else:
        z = r.standard_normal((N, d)) * np.exp(r.uniform(-3, 0, d))[None, :]
    return bf16_host(z.astype(np.float32))


# -------------------------------------------------------------- covariance
@pytest.mark.parametrize("N,d,kind", [(2048, 256, "t4"), (1000, 200, "g"), (4097, 520, "t4"),
                                      (130, 72, "g"), (64, 64, "t4"), (777, 1000, "g"),
                                      (20000, 384, "t4"), (33, 129, "g"), (70000, 256, "t4"),
                                      (8193, 136, "g"), (300, 257, "g"), (5000, 3104, "t4")])
def test_covariance_matches_oracle(cuda, N, d, kind):
    r = np.random.default_rng(N * 7 + d)
    lda = (d + 7) // 8 * 8                       # the ABI wants lda % 8 == 0
    bits = _x(r, N, lda, kind)
    ldh = (d + 3) // 4 * 4                       # and ldh % 4 == 0
    H = torch.full((d, ldh), float("nan"), device=cuda)[:, :d]
    abi.kronq_covariance(bf16_dev(bits, cuda)[:, :d], H, 1.0 / N, 0.0)
    Hg = H.cpu().numpy()
    ref = ocov.covariance(widen(bits)[:, :d])
    assert rel_fro(Hg, ref) <= 1e-4
    assert np.array_equal(Hg, Hg.T)
    np.testing.assert_allclose(np.diag(Hg), np.diag(ref), rtol=1e-4)


def test_covariance_padded_rows_beta_and_streaming(cuda):
    r = np.random.default_rng(5)
    N, d, pad = 3000, 264, 16
    bits = _x(r, N, d + pad, "t4")
    A = bf16_dev(bits, cuda)[:, :d]                 # lda = d + pad
    ref = ocov.covariance(widen(bits)[:, :d])
    # streamed over ragged chunks with alpha = 1/N, beta = 0 then 1
    H = torch.full((d, d), float("nan"), device=cuda)
    cuts = [0, 1000, 1001, 2500, N]
    for i in range(len(cuts) - 1):
        abi.kronq_covariance(A[cuts[i]:cuts[i + 1]], H, 1.0 / N, 0.0 if i == 0 else 1.0)
    assert rel_fro(H.cpu().numpy(), ref) <= 1e-4
    # beta != 0 with a symmetric start
    H0 = spd(r, d)
    H = t(H0, cuda)
    abi.kronq_covariance(A, H, 0.5 / N, 0.25)
    assert rel_fro(H.cpu().numpy(), 0.5 * ref + 0.25 * H0.astype(np.float64)) <= 1e-4
    # N = 0: H <- beta H
    H = t(H0, cuda)
    abi.kronq_covariance(A[:0], H, 1.0, 2.0)
    np.testing.assert_array_equal(H.cpu().numpy(), 2.0 * H0)


def test_covariance_shared_tiles_with_beta(cuda):
    """Enough tokens that CTA pairs split a tile's K range between them and
    add their parts into H (after the host-side scaling of H by beta)."""
    r = np.random.default_rng(11)
    N, d = 9000, 600
    bits = _x(r, N, d, "t4")
    A = bf16_dev(bits, cuda)
    ref = ocov.covariance(widen(bits))
    H0 = spd(r, d)
    for beta in (0.0, 0.25, 1.0):
        H = t(H0, cuda)
        abi.kronq_covariance(A, H, 1.0 / N, beta)
        want = ref + beta * H0.astype(np.float64)
        Hg = H.cpu().numpy()
        assert rel_fro(Hg, want) <= 1e-4, beta
        assert np.array_equal(Hg, Hg.T)


# ------------------------------------------------------------- sensitivity
def test_sensitivity_is_trace_product(cuda):
    r = np.random.default_rng(1)
    HX, HG = spd(r, 96), spd(r, 48)
    out = torch.zeros(3, dtype=torch.float64, device=cuda)
    abi.kronq_sensitivity(t(HX, cuda), t(HG, cuda), out)
    s, tx, tg = out.cpu().tolist()
    np.testing.assert_allclose(tx, np.trace(HX.astype(np.float64)), rtol=1e-12)
    np.testing.assert_allclose(tg, np.trace(HG.astype(np.float64)), rtol=1e-12)
    np.testing.assert_allclose(s, tx * tg, rtol=1e-14)


# -------------------------------------------------------------------- BiIP
def _biip_case(r, m, n):
    W = (r.standard_normal((m, n)) * 0.02 * np.exp(r.uniform(-1, 1, n))[None, :]).astype(np.float32)
    return W, spd(r, n), spd(r, m), signs(r, m), signs(r, n)


_BIIP_SHAPES = [(256, 256), (64, 112), (688, 96), (128, 448), (4096, 64), (112, 11008 // 8),
                (1024, 512), (2048, 128), (64, 2048)]


@pytest.mark.parametrize("m,n,mode", [(m, n, mode) for m, n in _BIIP_SHAPES
                                      for mode in ("full", "no_rescale", "su_only", "sv_only")]
                         + [(32, 8192, "full")])
def test_biip_matches_oracle(cuda, m, n, mode):
    r = np.random.default_rng(m + 3 * n)
    W, HX, HG, su, sv = _biip_case(r, m, n)
    Wd, HXd, HGd = t(W, cuda), t(HX, cuda), t(HG, cuda)
    SX = torch.empty(n, device=cuda)
    SG = torch.empty(m, device=cuda)
    ws = abi.workspace(m, n, device=cuda)
    abi.kronq_biip_rotate(Wd, HXd, HGd, t(su, cuda), t(sv, cuda), 0.25, mode, 0, SX, SG, ws)
    Wr, HXr, HGr, SXr, SGr = obiip.biip(W, HX, HG, su, sv, 0.25, mode)
    np.testing.assert_allclose(SX.cpu().numpy(), SXr, rtol=2e-6)
    np.testing.assert_allclose(SG.cpu().numpy(), SGr, rtol=2e-6)
    assert rel_fro(Wd.cpu().numpy(), Wr) <= 1e-5
    assert rel_fro(HXd.cpu().numpy(), HXr) <= 1e-5
    assert rel_fro(HGd.cpu().numpy(), HGr) <= 1e-5
    # exact inverse on W
    abi.kronq_biip_rotate(Wd, None, None, t(su, cuda), t(sv, cuda), 0.25, mode, 1, SX, SG, ws)
    assert rel_fro(Wd.cpu().numpy(), W) <= 1e-5


@pytest.mark.parametrize("m,n", [(64, 14336), (14336, 64), (32, 28672), (28672, 32)])
def test_biip_odd_factor_seven_wide(cuda, m, n):
    """Widths 7 x 2^11 and 7 x 2^12 (the LLaMA-3 MLP widths 14336 and 28672)
    take the fused passes: every segment's Walsh-Hadamard transform and the
    7-segment mix in one pass over the rows, and the column pass in two.
    Sampled entries of W', H_X', H_G' (64 x 64 blocks, every segment
    represented) and the scales in full, against the oracle."""
    r = np.random.default_rng(m + 5 * n)
    W = (r.standard_normal((m, n)) * 0.02 * np.exp(r.uniform(-1, 1, n))[None, :]).astype(np.float32)

    def wide(d):
        H = r.standard_normal((d, d), dtype=np.float32)
        H[np.arange(d), np.arange(d)] = np.abs(H[np.arange(d), np.arange(d)]) + 1.0
        return H

    HX, HG = wide(n), wide(m)
    su, sv = signs(r, m), signs(r, n)
    Wd, HXd, HGd = t(W, cuda), t(HX, cuda), t(HG, cuda)
    SX = torch.empty(n, device=cuda)
    SG = torch.empty(m, device=cuda)
    ws = abi.workspace(m, n, device=cuda)
    abi.kronq_biip_rotate(Wd, HXd, HGd, t(su, cuda), t(sv, cuda), 0.25, "full", 0, SX, SG, ws)
    torch.cuda.synchronize()
    pick = lambda d, k: np.sort(r.choice(d, min(d, k), replace=False))
    wr, wc, hxi, hgi = pick(m, 64), pick(n, 64), pick(n, 64), pick(m, 64)
    Wb, HXb, HGb, SXr, SGr = obiip.biip_entries(W, HX, HG, su, sv, 0.25, "full", wr, wc, hxi, hgi)
    np.testing.assert_allclose(SX.cpu().numpy(), SXr, rtol=2e-6)
    np.testing.assert_allclose(SG.cpu().numpy(), SGr, rtol=2e-6)
    assert rel_fro(Wd.cpu().numpy()[np.ix_(wr, wc)], Wb) <= 1e-5
    ix = torch.as_tensor(hxi, device=cuda)
    assert rel_fro(HXd[ix][:, ix].cpu().numpy(), HXb) <= 1e-5
    ig = torch.as_tensor(hgi, device=cuda)
    assert rel_fro(HGd[ig][:, ig].cpu().numpy(), HGb) <= 1e-5


@pytest.mark.parametrize("m,n", [(256, 256), (64, 112), (688, 96), (1024, 512), (112, 1376)])
@pytest.mark.parametrize("mode", ["full", "no_rescale", "su_only", "sv_only"])
def test_biip_alpha_half_matches_oracle(cuda, m, n, mode):
    """The weight-and-activation setting, --alpha 0.5 (KronQ README (GitHub),
    "Mapping paper results to flags"): the same kernels with the exponent
    1/2, against the oracle in every incoh mode."""
    r = np.random.default_rng(7 * m + n)
    W, HX, HG, su, sv = _biip_case(r, m, n)
    Wd, HXd, HGd = t(W, cuda), t(HX, cuda), t(HG, cuda)
    SX = torch.empty(n, device=cuda)
    SG = torch.empty(m, device=cuda)
    ws = abi.workspace(m, n, device=cuda)
    abi.kronq_biip_rotate(Wd, HXd, HGd, t(su, cuda), t(sv, cuda), 0.5, mode, 0, SX, SG, ws)
    Wr, HXr, HGr, SXr, SGr = obiip.biip(W, HX, HG, su, sv, 0.5, mode)
    np.testing.assert_allclose(SX.cpu().numpy(), SXr, rtol=2e-6)
    np.testing.assert_allclose(SG.cpu().numpy(), SGr, rtol=2e-6)
    assert rel_fro(Wd.cpu().numpy(), Wr) <= 1e-5
    assert rel_fro(HXd.cpu().numpy(), HXr) <= 1e-5
    assert rel_fro(HGd.cpu().numpy(), HGr) <= 1e-5


def test_biip_alpha_half_exchanges_diagonal_and_norms_on_gpu(cuda):
    """At alpha = 1/2 the input rescale swaps diag(H_X) and the squared
    column norms of W (closed form), checked on the GPU's own S_X: the
    rescaled diagonal H_jj / S_j^2 equals ||W_j||^2 and ||W_j||^2 S_j^2
    equals H_jj."""
    r = np.random.default_rng(23)
    m, n = 96, 512
    W, HX, HG, su, sv = _biip_case(r, m, n)
    SX = torch.empty(n, device=cuda)
    SG = torch.empty(m, device=cuda)
    ws = abi.workspace(m, n, device=cuda)
    abi.kronq_biip_rotate(t(W, cuda), t(HX, cuda), t(HG, cuda), t(su, cuda), t(sv, cuda), 0.5,
                          "sv_only", 0, SX, SG, ws)
    sx = SX.cpu().numpy().astype(np.float64)
    col2 = (W.astype(np.float64) ** 2).sum(0)
    hd = np.diag(HX).astype(np.float64)
    np.testing.assert_allclose(hd / sx ** 2, col2, rtol=1e-5)
    np.testing.assert_allclose(col2 * sx ** 2, hd, rtol=1e-5)


# ---------------------------------------------------------- inverse Cholesky
# n <= 1024 stays inside one 1024-wide super-block; 2304 and 3000 take outer
# (K = 1024) updates on fp16 row-scaled planes, 3000 also padding and a ragged
# last super-block
@pytest.mark.parametrize("n", [64, 72, 200, 256, 1000, 2304, 3000])
def test_cholesky_inv_matches_oracle(cuda, n):
    r = np.random.default_rng(n)
    H = spd(r, n, spread=1.5)
    U = torch.full((n, n), float("nan"), device=cuda)
    info = torch.zeros(1, dtype=torch.int32, device=cuda)
    ws = abi.workspace(n, n, device=cuda)
    abi.kronq_cholesky_inv(t(H, cuda), 0.01, U, info, ws)
    Ug = U.cpu().numpy().astype(np.float64)
    Uref = ochol.inverse_cholesky(ochol.damp(H, 0.01))
    assert info.item() == 0
    assert rel_fro(Ug, Uref) <= 1e-4
    assert np.all(np.tril(Ug, -1) == 0)
    Hd = ochol.damp(H, 0.01)
    assert rel_fro(Ug.T @ Ug @ Hd, np.eye(n)) <= 1e-4


def test_cholesky_flags_not_positive_definite(cuda):
    n = 96
    H = -np.eye(n, dtype=np.float32)
    U = torch.empty((n, n), device=cuda)
    info = torch.zeros(1, dtype=torch.int32, device=cuda)
    abi.kronq_cholesky_inv(t(H, cuda), 0.0, U, info, abi.workspace(n, n, device=cuda))
    torch.cuda.synchronize()
    assert info.item() == -3


# --------------------------------------------------------------- quantizer
@pytest.mark.parametrize("m,n,bits,group", [(256, 256, 4, -1), (100, 384, 2, 128),
                                            (37, 128, 3, -1), (64, 512, 2, 32), (300, 256, 4, 64),
                                            (128, 640, 8, -1), (130, 1024, 2, -1)])
def test_quantize_layer_matches_oracle(cuda, m, n, bits, group):
    r = np.random.default_rng(m * n + bits)
    W = (r.standard_normal((m, n)) * 0.02).astype(np.float32)
    U = ochol.inverse_cholesky(ochol.damp(spd(r, n, spread=1.0), 0.01)).astype(np.float32)
    G = 1 if group == -1 else n // group
    codes = torch.empty((m, n), dtype=torch.uint8, device=cuda)
    scales = torch.empty((m, G), device=cuda)
    zeros = torch.empty((m, G), dtype=torch.uint8, device=cuda)
    What = torch.empty((m, n), device=cuda)
    ws = abi.workspace(m, n, bits, group, device=cuda)
    abi.kronq_quantize_layer(t(W, cuda), t(U, cuda), bits, group, 128, codes, scales, zeros, What,
                             None, ws)
    ref = oq.obs_quantize(W, U, bits, group)
    cg = codes.cpu().numpy()
    same = (cg == ref["codes"]).mean()
    assert same >= 0.999, same
    if group == -1:
        np.testing.assert_array_equal(scales.cpu().numpy(), ref["scale"])
        np.testing.assert_array_equal(zeros.cpu().numpy(), ref["zero"])
    else:
        assert (zeros.cpu().numpy() == ref["zero"]).mean() >= 0.999
    Hd = np.linalg.inv(U.astype(np.float64).T @ U.astype(np.float64))
    lg = oq.row_losses(W - What.cpu().numpy(), Hd).sum()
    lr = oq.row_losses(W - ref["W_hat"], Hd).sum()
    assert abs(lg / lr - 1) <= 0.01
    # codes lie on the grid of their row / group
    assert cg.max() <= 2 ** bits - 1


# ------------------------------------------------------------------ packing
@pytest.mark.parametrize("m,n,bits", [(5, 96, 4), (7, 100, 4), (3, 17, 2), (64, 4096, 2), (1, 8, 4)])
def test_pack_unpack_bit_exact(cuda, m, n, bits):
    r = np.random.default_rng(m * n)
    codes = r.integers(0, 2 ** bits, (m, n), dtype=np.uint8)
    codes[0, : min(n, 2 ** bits)] = np.arange(min(n, 2 ** bits))
    packed = torch.full((m, abi.packed_words(n, bits)), -1, dtype=torch.int32, device=cuda)
    abi.kronq_pack(t(codes, cuda), bits, packed)
    ref = opack.pack(codes, bits)
    np.testing.assert_array_equal(packed.cpu().numpy().view(np.uint32), ref)
    back = torch.zeros((m, n), dtype=torch.uint8, device=cuda)
    abi.kronq_unpack(packed, n, bits, back)
    np.testing.assert_array_equal(back.cpu().numpy(), codes)


def test_pack_three_bit_unsupported(cuda):
    codes = torch.zeros((2, 32), dtype=torch.uint8, device=cuda)
    packed = torch.zeros((2, 3), dtype=torch.int32, device=cuda)
    with pytest.raises(abi.KronqError) as e:
        abi.kronq_pack(codes, 3, packed)
    assert e.value.code == -2


# ---------------------------------------------------------------- layer loss
def test_layer_loss_helper(cuda):
    r = np.random.default_rng(9)
    m, n = 96, 160
    Wr = r.standard_normal((m, n)).astype(np.float32)
    Wh = (Wr + 0.01 * r.standard_normal((m, n))).astype(np.float32)
    HX, HG = spd(r, n), spd(r, m)
    out = torch.zeros(1, dtype=torch.float64, device=cuda)
    abi.kronq_layer_loss(t(Wr, cuda), t(Wh, cuda), t(HX, cuda), t(HG, cuda), out,
                         abi.workspace(m, n, device=cuda))
    ref = oq.layer_loss(Wr.astype(np.float64) - Wh, HX, HG)
    np.testing.assert_allclose(out.item(), ref, rtol=1e-4)


# ------------------------------------------------------- failure detection
def test_bounded_wait_times_out_and_context_survives(cuda):
    info = torch.zeros(1, dtype=torch.int32, device=cuda)
    abi.kronq_selftest_wait(info, 20_000_000)      # 20 ms on a barrier nothing arrives on
    torch.cuda.synchronize()
    assert info.item() == -5
    # the context is still usable
    codes = torch.ones((2, 16), dtype=torch.uint8, device=cuda)
    packed = torch.zeros((2, 1), dtype=torch.int32, device=cuda)
    abi.kronq_pack(codes, 2, packed)
    torch.cuda.synchronize()
    assert packed[0, 0].item() == 0x55555555


def test_quantize_exact_ties_round_half_to_even(cuda):
    """Weights exactly on half-steps: the code decision (round half to even of
    the fp32 quotient) must match the oracle's bit for bit."""
    m, n = 4, 128
    W = np.zeros((m, n), dtype=np.float32)
    W[:, 0] = 0.0
    W[:, 1] = 15.0                                   # grid: lo 0, hi 15 -> scale 1, zero 0
    W[:, 2:32] = np.arange(30, dtype=np.float32)[None, :] * 0.5   # 0, 0.5, 1, ..., 14.5
    W[1] *= 0.25                                      # scale 0.25: exact multiples again
    W[2] *= -1.0                                      # lo -15: zero 15
    U = np.eye(n, dtype=np.float32)                   # no propagation: OBS == rounding
    codes = torch.empty((m, n), dtype=torch.uint8, device=cuda)
    scales = torch.empty((m, 1), device=cuda)
    zeros = torch.empty((m, 1), dtype=torch.uint8, device=cuda)
    abi.kronq_quantize_layer(t(W, cuda), t(U, cuda), 4, -1, 128, codes, scales, zeros, None, None,
                             abi.workspace(m, n, 4, -1, device=cuda))
    ref = oq.obs_quantize(W, U, 4, -1)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref["codes"])
    assert list(ref["codes"][0, 2:8]) == [0, 0, 1, 2, 2, 2]


def test_quantize_two_level_lazy_update_matches_one_level_and_oracle(cuda):
    """n = 2304 spans two full 1024-column super-blocks and a ragged one: the
    two-level lazy update (outer K = 1024 products) and the one-level update
    (chosen when the workspace only fits it) are both exact reassociations of
    the unblocked loop."""
    m, n, bits = 160, 2304, 4
    r = np.random.default_rng(77)
    W = (r.standard_normal((m, n)) * 0.02).astype(np.float32)
    U = ochol.inverse_cholesky(ochol.damp(spd(r, n, spread=1.0), 0.01)).astype(np.float32)
    ref = oq.obs_quantize(W, U, bits, -1)

    def a256(b):
        return (b + 255) // 256 * 256

    # the one-level scratch: E (m x 128) and the U_c slab (n x 128) as bf16 hi / lo planes
    one_level = 2 * a256(m * 128 * 2) + 2 * a256(n * 128 * 2)
    outs = []
    for ws in (abi.workspace(m, n, bits, -1, device=cuda),
               torch.empty(one_level, dtype=torch.uint8, device=cuda)):
        codes = torch.empty((m, n), dtype=torch.uint8, device=cuda)
        scales = torch.empty((m, 1), device=cuda)
        zeros = torch.empty((m, 1), dtype=torch.uint8, device=cuda)
        What = torch.empty((m, n), device=cuda)
        abi.kronq_quantize_layer(t(W, cuda), t(U, cuda), bits, -1, 128, codes, scales, zeros, What,
                                 None, ws)
        cg = codes.cpu().numpy()
        assert (cg == ref["codes"]).mean() >= 0.999
        outs.append((cg, What.cpu().numpy()))
    Hd = np.linalg.inv(U.astype(np.float64).T @ U.astype(np.float64))
    lr = oq.row_losses(W - ref["W_hat"], Hd).sum()
    for cg, wh in outs:
        assert abs(oq.row_losses(W - wh, Hd).sum() / lr - 1) <= 0.01
    assert (outs[0][0] == outs[1][0]).mean() >= 0.999
    # a workspace below the one-level size is refused
    with pytest.raises(abi.KronqError) as e:
        abi.kronq_quantize_layer(t(W, cuda), t(U, cuda), bits, -1, 128,
                                 torch.empty((m, n), dtype=torch.uint8, device=cuda),
                                 torch.empty((m, 1), device=cuda),
                                 torch.empty((m, 1), dtype=torch.uint8, device=cuda), None, None,
                                 torch.empty(one_level - 256, dtype=torch.uint8, device=cuda))
    assert e.value.code == -6
