"""Seeded generators for W, X, G and the rotation sign vectors.

Streams: numpy Philox (a counter-based generator) keyed by
key = (seed, tensor_id << 48 | index << 32 | chunk).  Token-major tensors are
drawn in chunks of CHUNK_TOKENS rows, each from its own key, so a chunk never
depends on another one.  Inside a chunk the rows are drawn in slabs of
SLAB_ROWS rows from the chunk's streams, in order; that order is part of the
definition of the data.

bf16 tensors are returned as uint16 bit patterns (round-to-nearest-even from
fp32); both sides widen them to their own working precision exactly.
"""

from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from .configs import Config, Sublayer, XSite

CHUNK_TOKENS = 16384
SLAB_ROWS = 1024

# tensor ids of the generator keys
T_W, T_X, T_G, T_SIGN_U, T_SIGN_V, T_OUTLIER, T_GSCALE, T_WROW, T_XAUX = 1, 2, 3, 4, 5, 6, 7, 8, 9
T_XDRIFT = 10

# Drift of the quantized model's layer input against the full-precision one
# (the asymmetric-calibration inputs): noise of this standard deviation per
# unit of the channel's scale.
DRIFT_SIGMA = 0.05


def _rng(seed: int, tensor_id: int, index: int, chunk: int = 0) -> np.random.Generator:
    k1 = (int(tensor_id) << 48) | (int(index) << 32) | int(chunk)
    return np.random.Generator(np.random.Philox(key=np.array([seed, k1], dtype=np.uint64)))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16 (nearest, ties to even); return the bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def n_chunks(tokens: int) -> int:
    return (tokens + CHUNK_TOKENS - 1) // CHUNK_TOKENS


def _threads(threads):
    return threads or max(1, min(32, os.cpu_count() or 1))


# ---------------------------------------------------------------- weights
def make_w(cfg: Config, sub: Sublayer) -> np.ndarray:
    """W (m x n) as fp32.  N(0, w_std^2); the toy layer scales each row's std
    by a log-uniform factor; the LLaMA-shaped layers hold bf16 values."""
    g = _rng(cfg.seed, T_W, sub.index)
    w = g.standard_normal((sub.m, sub.n), dtype=np.float32)
    w *= np.float32(cfg.w_std)
    if cfg.w_row_logrange is not None:
        lo, hi = cfg.w_row_logrange
        u = _rng(cfg.seed, T_WROW, sub.index).random(sub.m)
        f = np.exp(np.log(lo) + u * (np.log(hi) - np.log(lo))).astype(np.float32)
        w *= f[:, None]
    if cfg.w_round_bf16:
        w = bf16_bits_to_f32(f32_to_bf16_bits(w))
    return np.ascontiguousarray(w, dtype=np.float32)


def make_signs(cfg: Config, sub: Sublayer):
    """Random +-1 vectors for the output-side (length m) and input-side
    (length n) randomized Hadamard transforms, as int8."""
    su = _rng(cfg.seed, T_SIGN_U, sub.index).integers(0, 2, sub.m, dtype=np.int8)
    sv = _rng(cfg.seed, T_SIGN_V, sub.index).integers(0, 2, sub.n, dtype=np.int8)
    return (1 - 2 * su).astype(np.int8), (1 - 2 * sv).astype(np.int8)


# ------------------------------------------------------------ activations
def outlier_channels(cfg: Config, site: XSite) -> np.ndarray:
    k = cfg.outlier_count(site.width)
    perm = _rng(cfg.seed, T_OUTLIER, site.index).permutation(site.width)
    return np.sort(perm[:k])


def _chunk_rows(tokens: int, c: int) -> int:
    return min(CHUNK_TOKENS, tokens - c * CHUNK_TOKENS)


def x_chunk(cfg: Config, site: XSite, c: int, tokens: int | None = None,
            out: np.ndarray | None = None) -> np.ndarray:
    """Rows [c*CHUNK_TOKENS, ...) of X for one input site, as bf16 bits."""
    tokens = cfg.tokens if tokens is None else tokens
    rows = _chunk_rows(tokens, c)
    d = site.width
    if out is None:
        out = np.empty((rows, d), dtype=np.uint16)
    gz = _rng(cfg.seed, T_X, site.index, c)
    ga = _rng(cfg.seed, T_XAUX, site.index, c)
    oc = outlier_channels(cfg, site)
    slab = min(SLAB_ROWS, rows)
    z = np.empty((slab, d), dtype=np.float32)
    v = np.empty((slab, d), dtype=np.float32) if cfg.x_dist == "t4" else None
    for r0 in range(0, rows, SLAB_ROWS):
        r1 = min(rows, r0 + SLAB_ROWS)
        zz = z[: r1 - r0]
        gz.standard_normal(out=zz, dtype=np.float32)
        if cfg.x_dist == "t4":
            vv = v[: r1 - r0]
            # Student-t with 4 dof: z / sqrt(chi2_4 / 4), chi2_4 = 2 * Gamma(2)
            ga.standard_gamma(2.0, out=vv, dtype=np.float32)
            np.multiply(vv, np.float32(0.5), out=vv)
            np.sqrt(vv, out=vv)
            np.divide(zz, vv, out=zz)
        elif cfg.x_dist != "normal":
            raise ValueError(cfg.x_dist)
        if len(oc):
            zz[:, oc] *= np.float32(cfg.x_outlier_scale)
        out[r0:r1] = f32_to_bf16_bits(zz)
    return out


def xq_chunk(cfg: Config, site: XSite, c: int, tokens: int | None = None,
             sigma: float = DRIFT_SIGMA, out: np.ndarray | None = None,
             x_bits: np.ndarray | None = None) -> np.ndarray:
    """Rows [c*CHUNK_TOKENS, ...) of X~, the input the same site sees in the
    partly quantized model, as bf16 bits: the bf16 values of X plus seeded
    Gaussian noise of standard deviation sigma times the channel's scale
    (x_outlier_scale on the outlier channels, 1 elsewhere), rounded to bf16.
    x_bits: the same chunk of X when the caller has drawn it already."""
    xb = x_chunk(cfg, site, c, tokens) if x_bits is None else x_bits
    rows, d = xb.shape
    if out is None:
        out = np.empty((rows, d), dtype=np.uint16)
    scale = np.ones(d, dtype=np.float32)
    oc = outlier_channels(cfg, site)
    if len(oc):
        scale[oc] = np.float32(cfg.x_outlier_scale)
    gz = _rng(cfg.seed, T_XDRIFT, site.index, c)
    for r0 in range(0, rows, SLAB_ROWS):
        r1 = min(rows, r0 + SLAB_ROWS)
        z = gz.standard_normal((r1 - r0, d), dtype=np.float32)
        z *= np.float32(sigma) * scale[None, :]
        z += bf16_bits_to_f32(xb[r0:r1])
        out[r0:r1] = f32_to_bf16_bits(z)
    return out


def make_xq(cfg: Config, site: XSite, tokens: int | None = None, threads: int | None = None,
            sigma: float = DRIFT_SIGMA, out: np.ndarray | None = None) -> np.ndarray:
    """Whole X~ (tokens x width) for one site, bf16 bits."""
    tokens = cfg.tokens if tokens is None else tokens
    return _assemble(lambda c, o: xq_chunk(cfg, site, c, tokens, sigma, out=o), tokens,
                     site.width, threads, out)


def g_scales(cfg: Config, sub: Sublayer) -> np.ndarray:
    """Per-output-channel gradient scale 10^(-D u), u ~ U[0, 1)."""
    u = _rng(cfg.seed, T_GSCALE, sub.index).random(sub.m)
    return np.power(10.0, -cfg.g_decades * u).astype(np.float32)


def g_chunk(cfg: Config, sub: Sublayer, c: int, tokens: int | None = None,
            out: np.ndarray | None = None) -> np.ndarray:
    """Rows of the output gradient G (tokens x m) for one sublayer, bf16 bits."""
    tokens = cfg.tokens if tokens is None else tokens
    rows = _chunk_rows(tokens, c)
    m = sub.m
    if out is None:
        out = np.empty((rows, m), dtype=np.uint16)
    gz = _rng(cfg.seed, T_G, sub.index, c)
    sc = g_scales(cfg, sub)
    slab = min(SLAB_ROWS, rows)
    z = np.empty((slab, m), dtype=np.float32)
    for r0 in range(0, rows, SLAB_ROWS):
        r1 = min(rows, r0 + SLAB_ROWS)
        zz = z[: r1 - r0]
        gz.standard_normal(out=zz, dtype=np.float32)
        zz *= sc[None, :]
        out[r0:r1] = f32_to_bf16_bits(zz)
    return out


def _assemble(fn, tokens, width, threads, out=None):
    if out is None:
        out = np.empty((tokens, width), dtype=np.uint16)
    nc = n_chunks(tokens)

    def job(c):
        r0 = c * CHUNK_TOKENS
        fn(c, out[r0:r0 + _chunk_rows(tokens, c)])

    with ThreadPoolExecutor(_threads(threads)) as ex:
        list(ex.map(job, range(nc)))
    return out


def make_x(cfg: Config, site: XSite, tokens: int | None = None, threads: int | None = None,
           out: np.ndarray | None = None) -> np.ndarray:
    """Whole X (tokens x width) for one site, bf16 bits; chunks drawn in parallel."""
    tokens = cfg.tokens if tokens is None else tokens
    return _assemble(lambda c, o: x_chunk(cfg, site, c, tokens, out=o), tokens, site.width,
                     threads, out)


def make_g(cfg: Config, sub: Sublayer, tokens: int | None = None, threads: int | None = None,
           out: np.ndarray | None = None) -> np.ndarray:
    tokens = cfg.tokens if tokens is None else tokens
    return _assemble(lambda c, o: g_chunk(cfg, sub, c, tokens, out=o), tokens, sub.m,
                     threads, out)
