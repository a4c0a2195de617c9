"""The per-layer KronQ path as a sequence of libkronq calls on one stream.

Order (KronQ review (pith.science), appendix: Algorithm 1 then Algorithm 2;
KronQ summary (hyper.ai), "Method"):
  covariances -> BiIP -> sensitivity -> damped inverse Cholesky ->
  column-wise OBS quantization -> packing.

PyTorch only allocates device memory and provides streams here; every step
of the computation is a libkronq kernel.
"""

from __future__ import annotations

import contextlib
from dataclasses import dataclass

import torch

from . import abi
from .alloc import allocate_bits  # noqa: F401  (re-exported host logic)


@dataclass
class LayerResult:
    codes: torch.Tensor          # m x n uint8
    scales: torch.Tensor         # m x G fp32
    zeros: torch.Tensor          # m x G uint8
    packed: torch.Tensor | None  # m x words int32 (2- and 4-bit)
    sens: torch.Tensor           # 3 fp64 on device: s, tr(H_X'), tr(H_G')
    S_X: torch.Tensor
    S_G: torch.Tensor
    W_rot: torch.Tensor | None   # W' (kept when asked for)
    W_hat: torch.Tensor | None
    H_X: torch.Tensor            # rotated H_X'
    H_G: torch.Tensor            # rotated H_G'
    U_c: torch.Tensor            # factor of the (permuted, with act_order) damped H_X'
    info: torch.Tensor           # device int32 status word
    perm: torch.Tensor | None = None   # --act_order column order (int32), None without


def covariance(A: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """H = A^T A / N for a token-major bf16 matrix A (N x d) on the device."""
    N, d = A.shape
    H = out if out is not None else torch.empty((d, d), dtype=torch.float32, device=A.device)
    abi.kronq_covariance(A, H, 1.0 / max(N, 1), 0.0, stream=stream)
    return H


def quantize_sublayer(W: torch.Tensor, HX: torch.Tensor, HG: torch.Tensor,
                      sign_u: torch.Tensor, sign_v: torch.Tensor, bits: int, group: int = -1,
                      alpha: float = 0.25, mode: str = "full", damp: float = 0.01,
                      block: int = 128, keep: bool = False, ws: torch.Tensor | None = None,
                      in_place: bool = False, act_order: bool = False, clip: bool = False,
                      stream=None) -> LayerResult:
    """BiIP -> sensitivity -> inverse Cholesky -> OBS -> pack for one sublayer.

    W (m x n fp32), HX (n x n fp32), HG (m x m fp32) are device tensors.  They
    are cloned unless in_place is set (then W, HX, HG are overwritten).
    act_order / clip: the README's --act_order and --w_clip (readings in
    include/kronq.h); codes, W_hat and W_rot come back in the original column
    order, scales / zeros by groups of the permuted order.

    Every temporary is allocated while `stream` is the current stream, so the
    caching allocator ties its memory to the stream the kernels run on."""
    ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    with ctx:
        return _quantize_sublayer(W, HX, HG, sign_u, sign_v, bits, group, alpha, mode, damp, block,
                                  keep, ws, in_place, act_order, clip, stream)


def _quantize_sublayer(W, HX, HG, sign_u, sign_v, bits, group, alpha, mode, damp, block, keep, ws,
                       in_place, act_order, clip, stream) -> LayerResult:
    m, n = W.shape
    dev = W.device
    if not in_place:
        W, HX, HG = W.clone(), HX.clone(), HG.clone()
    if ws is None:
        ws = abi.workspace(m, n, bits, group, block, dev)
    info = torch.zeros(1, dtype=torch.int32, device=dev)
    SX = torch.empty(n, dtype=torch.float32, device=dev)
    SG = torch.empty(m, dtype=torch.float32, device=dev)
    abi.kronq_biip_rotate(W, HX, HG, sign_u, sign_v, alpha, mode, 0, SX, SG, ws, stream=stream)
    sens = torch.empty(3, dtype=torch.float64, device=dev)
    abi.kronq_sensitivity(HX, HG, sens, stream=stream)
    U = torch.empty((n, n), dtype=torch.float32, device=dev)
    W_rot = W.clone() if keep else None
    perm = None
    Hs, Ws = HX, W
    if act_order:
        perm = torch.empty(n, dtype=torch.int32, device=dev)
        abi.kronq_act_order(HX, perm, stream=stream)
        Hs, Ws = torch.empty_like(HX), torch.empty_like(W)
        abi.kronq_permute(HX, Hs, perm, abi.PERM_SYM, info, stream=stream)
        abi.kronq_permute(W, Ws, perm, abi.PERM_COLS, info, stream=stream)
    abi.kronq_cholesky_inv(Hs, damp, U, info, ws, stream=stream)
    G = 1 if group == -1 else n // group
    codes = torch.empty((m, n), dtype=torch.uint8, device=dev)
    scales = torch.empty((m, G), dtype=torch.float32, device=dev)
    zeros = torch.empty((m, G), dtype=torch.uint8, device=dev)
    W_hat = torch.empty((m, n), dtype=torch.float32, device=dev) if keep else None
    abi.kronq_quantize_layer_opt(Ws, U, bits, group, block, abi.QUANT_CLIP if clip else 0,
                                 codes, scales, zeros, W_hat, info, ws, stream=stream)
    if act_order:
        c_back = torch.empty_like(codes)
        abi.kronq_permute(codes, c_back, perm, abi.UNPERM_COLS, info, stream=stream)
        codes = c_back
        if W_hat is not None:
            h_back = torch.empty_like(W_hat)
            abi.kronq_permute(W_hat, h_back, perm, abi.UNPERM_COLS, info, stream=stream)
            W_hat = h_back
    packed = None
    if bits in (2, 4):
        packed = torch.empty((m, abi.packed_words(n, bits)), dtype=torch.int32, device=dev)
        abi.kronq_pack(codes, bits, packed, stream=stream)
    return LayerResult(codes, scales, zeros, packed, sens, SX, SG, W_rot, W_hat, HX, HG, U, info,
                       perm)


def covariance_from_host(A_host: torch.Tensor, H: torch.Tensor, chunk_rows: int = 16384,
                         copy_stream=None, stream=None, staging=None) -> int:
    """Stream a pinned host bf16 matrix through two device staging buffers:
    the copy of chunk c+1 overlaps the covariance of chunk c.  Returns the
    bytes copied host -> device."""
    N, d = A_host.shape
    dev = H.device
    stream = stream or torch.cuda.current_stream(dev)
    copy_stream = copy_stream or torch.cuda.Stream(dev)
    if staging is None:
        # allocated on the compute stream and also used by the copy stream
        with torch.cuda.stream(stream):
            staging = [torch.empty((chunk_rows, d), dtype=torch.bfloat16, device=dev)
                       for _ in range(2)]
        for t in staging:
            t.record_stream(copy_stream)
    done = [torch.cuda.Event(), torch.cuda.Event()]
    used = [torch.cuda.Event(), torch.cuda.Event()]
    nchunks = (N + chunk_rows - 1) // chunk_rows
    if nchunks == 0:
        with torch.cuda.stream(stream):
            abi.kronq_covariance(A_host[:0].to(dev), H, 0.0, 0.0, stream=stream)
        return 0
    copied = 0
    for c in range(nchunks):
        b = c & 1
        r0, r1 = c * chunk_rows, min(N, (c + 1) * chunk_rows)
        with torch.cuda.stream(copy_stream):
            if c >= 2:
                copy_stream.wait_event(used[b])
            staging[b][: r1 - r0].copy_(A_host[r0:r1], non_blocking=True)
            done[b].record(copy_stream)
        copied += (r1 - r0) * d * 2
        stream.wait_event(done[b])
        abi.kronq_covariance(staging[b][: r1 - r0], H, 1.0 / N, 0.0 if c == 0 else 1.0, stream=stream)
        used[b].record(stream)
    return copied


@dataclass
class GptaqResult:
    codes: torch.Tensor
    scales: torch.Tensor
    zeros: torch.Tensor
    packed: torch.Tensor | None
    S_X: torch.Tensor
    S_G: torch.Tensor
    W_rot: torch.Tensor | None
    W_hat: torch.Tensor | None
    H_X: torch.Tensor            # rotated covariance of the drifted input X~
    H_G: torch.Tensor
    A: torch.Tensor              # rotated drift covariance (X - X~)^T X~ / N
    U_c: torch.Tensor
    P: torch.Tensor
    info: torch.Tensor


def quantize_sublayer_gptaq(W: torch.Tensor, HX: torch.Tensor, A: torch.Tensor, HG: torch.Tensor,
                            sign_u: torch.Tensor, sign_v: torch.Tensor, bits: int, group: int = -1,
                            alpha: float = 0.25, mode: str = "full", damp: float = 0.01,
                            block: int = 128, alpha_asym: float = 0.25, keep: bool = False,
                            ws: torch.Tensor | None = None, stream=None) -> GptaqResult:
    """The layer path with GPTAQ's asymmetric calibration: HX = X~^T X~ / N and
    A = (X - X~)^T X~ / N (kronq_drift_covariance), HG = G^T G / N.  BiIP ->
    the drift covariance rotated like H_X -> inverse Cholesky -> P -> the
    column loop with the P term -> pack.  Inputs are cloned."""
    ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    with ctx:
        m, n = W.shape
        dev = W.device
        W, HX, A, HG = W.clone(), HX.clone(), A.clone(), HG.clone()
        if ws is None:
            ws = abi.gptaq_workspace(m, n, dev)
        info = torch.zeros(1, dtype=torch.int32, device=dev)
        SX = torch.empty(n, dtype=torch.float32, device=dev)
        SG = torch.empty(m, dtype=torch.float32, device=dev)
        abi.kronq_biip_rotate(W, HX, HG, sign_u, sign_v, alpha, mode, 0, SX, SG, ws, stream=stream)
        abi.kronq_biip_rotate_input(A, SX, sign_v, mode, ws, stream=stream)
        U = torch.empty((n, n), dtype=torch.float32, device=dev)
        abi.kronq_cholesky_inv(HX, damp, U, info, ws, stream=stream)
        P = torch.empty((n, n), dtype=torch.float32, device=dev)
        abi.kronq_gptaq_correction(A, U, alpha_asym, P, info, ws, stream=stream)
        W_rot = W.clone() if keep else None
        G = 1 if group == -1 else n // group
        codes = torch.empty((m, n), dtype=torch.uint8, device=dev)
        scales = torch.empty((m, G), dtype=torch.float32, device=dev)
        zeros = torch.empty((m, G), dtype=torch.uint8, device=dev)
        W_hat = torch.empty((m, n), dtype=torch.float32, device=dev) if keep else None
        abi.kronq_quantize_layer_gptaq(W, U, P, bits, group, block, codes, scales, zeros, W_hat,
                                       info, ws, stream=stream)
        packed = None
        if bits in (2, 4):
            packed = torch.empty((m, abi.packed_words(n, bits)), dtype=torch.int32, device=dev)
            abi.kronq_pack(codes, bits, packed, stream=stream)
        return GptaqResult(codes, scales, zeros, packed, SX, SG, W_rot, W_hat, HX, HG, A, U, P, info)
