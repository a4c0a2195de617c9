"""Python binding of libkronq: the C ABI of include/kronq.h, one function per
entry point, same names.  Argument marshalling only (device pointers, sizes,
the current CUDA stream); every computation runs in the CUDA library.

There is no fallback: if libkronq.so is missing or fails to load, every call
raises.
"""

from __future__ import annotations

import ctypes
import pathlib

import torch

HERE = pathlib.Path(__file__).resolve().parent
LIB_PATH = HERE / "libkronq.so"

KRONQ_OK = 0
STATUS = {
    0: "ok", -1: "invalid argument", -2: "unsupported", -3: "matrix not positive definite",
    -4: "CUDA error", -5: "device wait timed out", -6: "workspace missing or too small",
}
MODES = {"full": 0, "no_rescale": 1, "su_only": 2, "sv_only": 3}
QUANT_CLIP = 1                      # kronq_quantize_layer_opt options
PERM_COLS, UNPERM_COLS, PERM_SYM = 0, 1, 2   # kronq_permute modes

_lib = None


class KronqError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {STATUS.get(code, 'unknown status')} ({code})")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load libkronq.so (built in-tree by post_quantization_02_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not LIB_PATH.exists():
        raise RuntimeError(f"{LIB_PATH} is not built; run `python -m post_quantization_02_b200.build`")
    L = ctypes.CDLL(str(LIB_PATH))
    P, I64, I32, F32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "kronq_status_string": ([I32], ctypes.c_char_p),
        "kronq_abi_version": ([], I32),
        "kronq_launch_count": ([], ctypes.c_uint64),
        "kronq_workspace_size": ([I64, I64, I32, I32, I32], SZ),
        "kronq_covariance": ([P, I64, I64, I64, P, I64, F32, F32, P, P], I32),
        "kronq_sensitivity": ([P, I64, P, I64, P, P], I32),
        "kronq_biip_rotate": ([P, I64, I64, P, P, P, P, F32, I32, I32, P, P, P, SZ, P], I32),
        "kronq_cholesky_inv": ([P, I64, F32, P, P, P, SZ, P], I32),
        "kronq_quantize_layer": ([P, I64, I64, P, I32, I32, I32, P, P, P, P, P, P, SZ, P], I32),
        "kronq_quantize_layer_noalloc": ([P, I64, I64, P, I32, I32, I32, P, P, P, P, P, P], I32),
        "kronq_quantize_layer_opt": ([P, I64, I64, P, I32, I32, I32, I32, P, P, P, P, P, P, SZ, P], I32),
        "kronq_act_order": ([P, I64, P, P], I32),
        "kronq_permute": ([P, P, I64, I64, I32, P, I32, P, P], I32),
        "kronq_deploy_workspace_size": ([I64, I64, I64], SZ),
        "kronq_deploy_matvec": ([P, I64, I64, I32, I32, P, P, P, P, P, P, I32, P, I64, P, P, SZ, P], I32),
        "kronq_pack": ([P, I64, I64, I32, P, P], I32),
        "kronq_unpack": ([P, I64, I64, I32, P, P], I32),
        "kronq_layer_loss": ([P, P, I64, I64, P, P, P, P, SZ, P], I32),
        "kronq_selftest_wait": ([P, I64, P], I32),
        "kronq_sync_status": ([P, P], I32),
        "kronq_gptaq_workspace_size": ([I64, I64], SZ),
        "kronq_drift_covariance": ([P, I64, I64, I64, P, P, P, P, SZ, P], I32),
        "kronq_biip_rotate_input": ([P, I64, P, P, I32, P, SZ, P], I32),
        "kronq_gptaq_correction": ([P, P, I64, F32, P, P, P, SZ, P], I32),
        "kronq_quantize_layer_gptaq": ([P, I64, I64, P, P, I32, I32, I32, P, P, P, P, P, P, SZ, P], I32),
        "kronq_timing_enable": ([I32], I32),
        "kronq_timing_read": ([I32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_uint64)], I32),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, code: int):
    if code != KRONQ_OK:
        raise KronqError(fn, code)


def _dev(t, dtype, name, ndim=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a torch tensor")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


def _shape(t, shape, name):
    """t must have exactly this shape (None: no tensor given, nothing to check)."""
    if t is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _numel(t, count, name):
    if t is not None and t.numel() != count:
        raise ValueError(f"{name} has {t.numel()} elements, expected {count}")


def _on_current_device(*named):
    """Every tensor lives on the current CUDA device: the kernels launch there
    (and per-device library state is looked up there)."""
    tensors = [(t, nm) for t, nm in named if t is not None]
    for t, nm in tensors:
        if not t.is_cuda:
            raise ValueError(f"{nm} must be a CUDA tensor")
    if tensors:
        cur = torch.cuda.current_device()
        for t, nm in tensors:
            if t.device.index != cur:
                raise ValueError(f"{nm} is on cuda:{t.device.index}, the current device is cuda:{cur}")


def _contig(t, name):
    if t is not None and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _groups(n: int, group: int) -> int:
    return 1 if group == -1 or group <= 0 else max(1, n // group)


def _quant_args(W, U, codes, scales, zeros, W_hat, group):
    """Types, shapes and placement of the solver's tensors for an m x n layer."""
    _dev(W, torch.float32, "W", 2)
    _dev(U, torch.float32, "U_c", 2)
    _dev(codes, torch.uint8, "codes", 2)
    _dev(scales, torch.float32, "scales")
    _dev(zeros, torch.uint8, "zeros")
    _dev(W_hat, torch.float32, "W_hat", 2)
    m, n = W.shape
    G = _groups(n, group)
    _shape(U, (n, n), "U_c")
    _shape(codes, (m, n), "codes")
    _numel(scales, m * G, "scales")
    _numel(zeros, m * G, "zeros")
    _shape(W_hat, (m, n), "W_hat")
    named = ((W, "W"), (U, "U_c"), (codes, "codes"), (scales, "scales"), (zeros, "zeros"),
             (W_hat, "W_hat"))
    _on_current_device(*named)
    for t, nm in named:
        _contig(t, nm)
    return m, n


def kronq_status_string(code: int) -> str:
    return lib().kronq_status_string(code).decode()


def kronq_abi_version() -> int:
    return lib().kronq_abi_version()


def kronq_launch_count() -> int:
    return int(lib().kronq_launch_count())


def kronq_workspace_size(m: int, n: int, bits: int = 4, group: int = -1, block: int = 128) -> int:
    return int(lib().kronq_workspace_size(m, n, bits, group, block))


def workspace(m: int, n: int, bits: int = 4, group: int = -1, block: int = 128, device=None):
    """A caller-owned workspace tensor of kronq_workspace_size bytes."""
    nbytes = kronq_workspace_size(m, n, bits, group, block)
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device or "cuda")


def kronq_covariance(A, H, alpha: float, beta: float = 0.0, info=None, stream=None):
    """H = alpha A^T A + beta H.  A: (N, d) bf16 (row stride lda, unit column
    stride); H: (d, d) fp32 with unit column stride."""
    _dev(A, (torch.bfloat16, torch.int16, torch.uint16), "A", 2)
    _dev(H, torch.float32, "H", 2)
    _dev(info, torch.int32, "info")
    N, d = A.shape
    _shape(H, (d, d), "H")
    _on_current_device((A, "A"), (H, "H"), (info, "info"))
    if A.stride(1) != 1 or H.stride(1) != 1:
        raise ValueError("A and H need unit stride along their last dimension")
    _check("kronq_covariance", lib().kronq_covariance(
        _p(A), N, d, A.stride(0) if N > 0 else d, _p(H), H.stride(0), alpha, beta, _p(info), _s(stream)))


def kronq_sensitivity(HX, HG, out, stream=None):
    """out (3 fp64, device) = {tr(H_G) tr(H_X), tr(H_X), tr(H_G)}."""
    _dev(HX, torch.float32, "H_X", 2)
    _dev(HG, torch.float32, "H_G", 2)
    _dev(out, torch.float64, "out")
    _shape(HX, (HX.shape[0], HX.shape[0]), "H_X")
    _shape(HG, (HG.shape[0], HG.shape[0]), "H_G")
    if out.numel() < 3:
        raise ValueError("out needs 3 fp64 elements")
    _on_current_device((HX, "H_X"), (HG, "H_G"), (out, "out"))
    _contig(HX, "H_X"); _contig(HG, "H_G")
    _check("kronq_sensitivity", lib().kronq_sensitivity(
        _p(HX), HX.shape[0], _p(HG), HG.shape[0], _p(out), _s(stream)))


def kronq_biip_rotate(W, HX, HG, sign_u, sign_v, alpha: float, mode, inverse: int, SX, SG, ws,
                      stream=None):
    _dev(W, torch.float32, "W", 2)
    _dev(HX, torch.float32, "H_X", 2)
    _dev(HG, torch.float32, "H_G", 2)
    _dev(sign_u, torch.int8, "sign_u")
    _dev(sign_v, torch.int8, "sign_v")
    _dev(SX, torch.float32, "S_X")
    _dev(SG, torch.float32, "S_G")
    _dev(ws, None, "ws")
    m, n = W.shape
    _shape(HX, (n, n), "H_X")
    _shape(HG, (m, m), "H_G")
    _numel(sign_u, m, "sign_u")
    _numel(sign_v, n, "sign_v")
    _numel(SX, n, "S_X")
    _numel(SG, m, "S_G")
    named = ((W, "W"), (HX, "H_X"), (HG, "H_G"), (sign_u, "sign_u"), (sign_v, "sign_v"),
             (SX, "S_X"), (SG, "S_G"), (ws, "ws"))
    _on_current_device(*named)
    for t, nm in named:
        _contig(t, nm)
    mode = MODES[mode] if isinstance(mode, str) else int(mode)
    _check("kronq_biip_rotate", lib().kronq_biip_rotate(
        _p(W), m, n, _p(HX), _p(HG), _p(sign_u), _p(sign_v), alpha, mode, int(inverse),
        _p(SX), _p(SG), _p(ws), 0 if ws is None else ws.numel() * ws.element_size(), _s(stream)))


def kronq_cholesky_inv(H, damp_rel: float, U, info, ws, stream=None):
    _dev(H, torch.float32, "H", 2)
    _dev(U, torch.float32, "U_c", 2)
    _dev(info, torch.int32, "info")
    _dev(ws, None, "ws")
    n = H.shape[0]
    _shape(H, (n, n), "H")
    _shape(U, (n, n), "U_c")
    _on_current_device((H, "H"), (U, "U_c"), (info, "info"), (ws, "ws"))
    _contig(H, "H"); _contig(U, "U_c"); _contig(ws, "ws")
    _check("kronq_cholesky_inv", lib().kronq_cholesky_inv(
        _p(H), n, damp_rel, _p(U), _p(info), _p(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _s(stream)))


def kronq_quantize_layer(W, U, bits: int, group: int, block: int, codes, scales, zeros,
                         W_hat=None, info=None, ws=None, stream=None):
    m, n = _quant_args(W, U, codes, scales, zeros, W_hat, group)
    _dev(info, torch.int32, "info")
    _dev(ws, None, "ws")
    _on_current_device((info, "info"), (ws, "ws"))
    _check("kronq_quantize_layer", lib().kronq_quantize_layer(
        _p(W), m, n, _p(U), bits, group, block, _p(codes), _p(scales), _p(zeros), _p(W_hat),
        _p(info), _p(ws), 0 if ws is None else ws.numel() * ws.element_size(), _s(stream)))


def kronq_quantize_layer_opt(W, U, bits: int, group: int, block: int, options: int, codes, scales,
                             zeros, W_hat=None, info=None, ws=None, stream=None):
    """kronq_quantize_layer with option flags (QUANT_CLIP: the --w_clip search)."""
    m, n = _quant_args(W, U, codes, scales, zeros, W_hat, group)
    _dev(info, torch.int32, "info")
    _dev(ws, None, "ws")
    _on_current_device((info, "info"), (ws, "ws"))
    _check("kronq_quantize_layer_opt", lib().kronq_quantize_layer_opt(
        _p(W), m, n, _p(U), bits, group, block, options, _p(codes), _p(scales), _p(zeros),
        _p(W_hat), _p(info), _p(ws), 0 if ws is None else ws.numel() * ws.element_size(),
        _s(stream)))


def kronq_act_order(H, perm, stream=None):
    """perm (int32, n) = the --act_order column order from diag(H)."""
    _dev(H, torch.float32, "H", 2)
    _dev(perm, torch.int32, "perm", 1)
    n = H.shape[0]
    _shape(H, (n, n), "H")
    _numel(perm, n, "perm")
    _on_current_device((H, "H"), (perm, "perm"))
    _contig(H, "H")
    _check("kronq_act_order", lib().kronq_act_order(_p(H), n, _p(perm), _s(stream)))


def kronq_permute(src, dst, perm, mode: int, info=None, stream=None):
    """Column / symmetric permutation of a 2-D uint8 or fp32 tensor (see kronq.h)."""
    _dev(src, (torch.float32, torch.uint8), "src", 2)
    _dev(dst, src.dtype, "dst", 2)
    _dev(perm, torch.int32, "perm", 1)
    _dev(info, torch.int32, "info")
    if dst.shape != src.shape or perm.numel() != src.shape[1]:
        raise ValueError("kronq_permute: shapes do not match")
    _on_current_device((src, "src"), (dst, "dst"), (perm, "perm"), (info, "info"))
    _contig(src, "src"); _contig(dst, "dst")
    m, n = src.shape
    _check("kronq_permute", lib().kronq_permute(_p(src), _p(dst), m, n, src.element_size(),
                                                _p(perm), mode, _p(info), _s(stream)))


def kronq_deploy_workspace_size(m: int, n: int, batch: int) -> int:
    return lib().kronq_deploy_workspace_size(m, n, batch)


def deploy_workspace(m: int, n: int, batch: int, device=None) -> torch.Tensor:
    nbytes = kronq_deploy_workspace_size(m, n, batch)
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def kronq_deploy_matvec(packed, n: int, bits: int, group: int, scales, zeros, SX, SG, sign_u, sign_v,
                        mode, x, y, ws, stream=None):
    """y (batch x m) = W_hat x for x (batch x n) from the packed layer (see kronq.h)."""
    _dev(packed, (torch.int32, torch.uint32), "packed", 2)
    _dev(x, torch.float32, "x", 2)
    _dev(y, torch.float32, "y", 2)
    _dev(scales, torch.float32, "scales")
    _dev(zeros, torch.uint8, "zeros")
    _dev(SX, torch.float32, "S_X")
    _dev(SG, torch.float32, "S_G")
    _dev(sign_u, torch.int8, "sign_u")
    _dev(sign_v, torch.int8, "sign_v")
    m = packed.shape[0]
    batch = x.shape[0]
    if x.shape[1] != n or y.shape != (batch, m):
        raise ValueError("kronq_deploy_matvec: shapes do not match")
    G = _groups(n, group)
    _shape(packed, (m, packed_words(n, bits)), "packed")
    _numel(scales, m * G, "scales")
    _numel(zeros, m * G, "zeros")
    _numel(SX, n, "S_X")
    _numel(SG, m, "S_G")
    _numel(sign_u, m, "sign_u")
    _numel(sign_v, n, "sign_v")
    named = ((packed, "packed"), (scales, "scales"), (zeros, "zeros"), (SX, "S_X"), (SG, "S_G"),
             (sign_u, "sign_u"), (sign_v, "sign_v"), (x, "x"), (y, "y"), (ws, "ws"))
    _on_current_device(*named)
    for t_, nm in named:
        _contig(t_, nm)
    md = MODES[mode] if isinstance(mode, str) else int(mode)
    _check("kronq_deploy_matvec", lib().kronq_deploy_matvec(
        _p(packed), m, n, bits, group, _p(scales), _p(zeros), _p(SX), _p(SG), _p(sign_u),
        _p(sign_v), md, _p(x), batch, _p(y), _p(ws), ws.numel() * ws.element_size(), _s(stream)))


def kronq_quantize_layer_noalloc(W, U, bits: int, group: int, block: int, codes, scales, zeros,
                                 W_hat=None, info=None, stream=None):
    """kronq_quantize_layer with its scratch in the library's static device
    array (no workspace, nothing allocated; at most 32768 rows and 32768
    columns).  Layers whose two-level lazy-update scratch exceeds the array's
    64 MiB (e.g. 8192 x 8192) run the one-level update (K = 128 trailing
    updates): the same codes up to floating-point summation order, at a
    lower speed."""
    m, n = _quant_args(W, U, codes, scales, zeros, W_hat, group)
    _dev(info, torch.int32, "info")
    _on_current_device((info, "info"))
    _check("kronq_quantize_layer_noalloc", lib().kronq_quantize_layer_noalloc(
        _p(W), m, n, _p(U), bits, group, block, _p(codes), _p(scales), _p(zeros), _p(W_hat),
        _p(info), _s(stream)))


def kronq_pack(codes, bits: int, packed, stream=None):
    _dev(codes, torch.uint8, "codes", 2)
    _dev(packed, (torch.int32, torch.uint32), "packed", 2)
    m, n = codes.shape
    if bits in (2, 4):
        _shape(packed, (m, packed_words(n, bits)), "packed")
    _on_current_device((codes, "codes"), (packed, "packed"))
    _contig(codes, "codes"); _contig(packed, "packed")
    _check("kronq_pack", lib().kronq_pack(_p(codes), m, n, bits, _p(packed), _s(stream)))


def kronq_unpack(packed, n: int, bits: int, codes, stream=None):
    _dev(codes, torch.uint8, "codes", 2)
    _dev(packed, (torch.int32, torch.uint32), "packed", 2)
    m = codes.shape[0]
    _shape(codes, (m, n), "codes")
    if bits in (2, 4):
        _shape(packed, (m, packed_words(n, bits)), "packed")
    _on_current_device((codes, "codes"), (packed, "packed"))
    _contig(codes, "codes"); _contig(packed, "packed")
    _check("kronq_unpack", lib().kronq_unpack(_p(packed), m, n, bits, _p(codes), _s(stream)))


def kronq_layer_loss(W_ref, W_hat, HX, HG, out, ws, stream=None):
    for t, nm in ((W_ref, "W_ref"), (W_hat, "W_hat"), (HX, "H_X"), (HG, "H_G")):
        _dev(t, torch.float32, nm, 2)
    _dev(out, torch.float64, "loss_out")
    m, n = W_ref.shape
    _shape(W_hat, (m, n), "W_hat")
    _shape(HX, (n, n), "H_X")
    _shape(HG, (m, m), "H_G")
    named = ((W_ref, "W_ref"), (W_hat, "W_hat"), (HX, "H_X"), (HG, "H_G"), (out, "loss_out"),
             (ws, "ws"))
    _on_current_device(*named)
    for t, nm in named[:4]:
        _contig(t, nm)
    _check("kronq_layer_loss", lib().kronq_layer_loss(
        _p(W_ref), _p(W_hat), m, n, _p(HX), _p(HG), _p(out), _p(ws),
        ws.numel() * ws.element_size(), _s(stream)))


# ------------------------------------------------ GPTAQ asymmetric calibration
def kronq_gptaq_workspace_size(m: int, n: int) -> int:
    return int(lib().kronq_gptaq_workspace_size(m, n))


def gptaq_workspace(m: int, n: int, device=None):
    return torch.empty(max(kronq_gptaq_workspace_size(m, n), 256), dtype=torch.uint8,
                       device=device or "cuda")


def kronq_drift_covariance(XqX, H, A, info=None, ws=None, stream=None):
    """H = X~^T X~ / N, A = (X - X~)^T X~ / N from XqX = [X~ | X] (N x 2n bf16)."""
    _dev(XqX, (torch.bfloat16, torch.int16, torch.uint16), "XqX", 2)
    _dev(H, torch.float32, "H", 2)
    _dev(A, torch.float32, "A", 2)
    _dev(info, torch.int32, "info")
    N, w2 = XqX.shape
    if w2 % 2:
        raise ValueError("XqX must have an even width (X~ then X)")
    n = w2 // 2
    _shape(H, (n, n), "H")
    _shape(A, (n, n), "A")
    _on_current_device((XqX, "XqX"), (H, "H"), (A, "A"), (info, "info"), (ws, "ws"))
    if XqX.stride(1) != 1:
        raise ValueError("XqX needs unit stride along its last dimension")
    _contig(H, "H"); _contig(A, "A")
    _check("kronq_drift_covariance", lib().kronq_drift_covariance(
        _p(XqX), N, n, XqX.stride(0) if N > 0 else w2, _p(H), _p(A), _p(info), _p(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _s(stream)))


def kronq_biip_rotate_input(A, SX, sign_v, mode, ws, stream=None):
    _dev(A, torch.float32, "A", 2)
    _dev(SX, torch.float32, "S_X")
    _dev(sign_v, torch.int8, "sign_v")
    n = A.shape[0]
    _shape(A, (n, n), "A")
    _numel(SX, n, "S_X")
    _numel(sign_v, n, "sign_v")
    _on_current_device((A, "A"), (SX, "S_X"), (sign_v, "sign_v"), (ws, "ws"))
    _contig(A, "A")
    md = MODES[mode] if isinstance(mode, str) else int(mode)
    _check("kronq_biip_rotate_input", lib().kronq_biip_rotate_input(
        _p(A), n, _p(SX), _p(sign_v), md, _p(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _s(stream)))


def kronq_gptaq_correction(A, U, alpha: float, P, info=None, ws=None, stream=None):
    for t, nm in ((A, "A"), (U, "U_c"), (P, "P")):
        _dev(t, torch.float32, nm, 2)
    n = A.shape[0]
    for t, nm in ((A, "A"), (U, "U_c"), (P, "P")):
        _shape(t, (n, n), nm)
    _dev(info, torch.int32, "info")
    _on_current_device((A, "A"), (U, "U_c"), (P, "P"), (info, "info"), (ws, "ws"))
    for t, nm in ((A, "A"), (U, "U_c"), (P, "P")):
        _contig(t, nm)
    _check("kronq_gptaq_correction", lib().kronq_gptaq_correction(
        _p(A), _p(U), n, alpha, _p(P), _p(info), _p(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _s(stream)))


def kronq_quantize_layer_gptaq(W, U, P, bits: int, group: int, block: int, codes, scales, zeros,
                               W_hat=None, info=None, ws=None, stream=None):
    m, n = _quant_args(W, U, codes, scales, zeros, W_hat, group)
    _dev(P, torch.float32, "P", 2)
    _shape(P, (n, n), "P")
    _dev(info, torch.int32, "info")
    _on_current_device((P, "P"), (info, "info"), (ws, "ws"))
    _contig(P, "P")
    _check("kronq_quantize_layer_gptaq", lib().kronq_quantize_layer_gptaq(
        _p(W), m, n, _p(U), _p(P), bits, group, block, _p(codes), _p(scales), _p(zeros),
        _p(W_hat), _p(info), _p(ws), 0 if ws is None else ws.numel() * ws.element_size(),
        _s(stream)))


TIMERS = {"lazy_update": 0, "chol_update": 1, "chol_panel": 2, "obs_block": 3}


def kronq_timing_enable(on: bool = True):
    """Start (and clear) or stop the library's event timing of its inner launches."""
    _check("kronq_timing_enable", lib().kronq_timing_enable(1 if on else 0))


def kronq_timing_read(category) -> tuple:
    """(summed device ms, launches) of one timer category on the current device."""
    cat = TIMERS[category] if isinstance(category, str) else int(category)
    ms = ctypes.c_double(0.0)
    cnt = ctypes.c_uint64(0)
    _check("kronq_timing_read", lib().kronq_timing_read(cat, ctypes.byref(ms), ctypes.byref(cnt)))
    return ms.value, int(cnt.value)


def kronq_selftest_wait(info, limit_ns: int, stream=None):
    _dev(info, torch.int32, "info")
    _on_current_device((info, "info"))
    _check("kronq_selftest_wait", lib().kronq_selftest_wait(_p(info), int(limit_ns), _s(stream)))


def kronq_sync_status(stream=None, info=None) -> int:
    """Wait for `stream` and return its status: KRONQ_ERR_CUDA (-4) after a
    CUDA error, else the device word `info` (0 or the first numerical
    failure), else 0.  Returns the code rather than raising."""
    _dev(info, torch.int32, "info")
    return int(lib().kronq_sync_status(_s(stream), _p(info)))


def packed_words(n: int, bits: int) -> int:
    return (n * bits + 31) // 32
