"""The C ABI: libkronq.so loads, exports every symbol include/kronq.h
declares, and rejects bad arguments on the host (no kernel is launched by any
call here; these run without a GPU)."""

import ctypes
import re

import pytest

from conftest import ROOT

HEADER = ROOT / "include" / "kronq.h"


def _declared():
    text = re.sub(r"/\*.*?\*/", "", HEADER.read_text(), flags=re.S)
    return sorted(set(re.findall(r"\b(kronq_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    from post_quantization_02_b200 import build, abi
    build.build()
    return abi.lib()


def test_header_declares_the_path():
    names = _declared()
    for required in ("kronq_covariance", "kronq_sensitivity", "kronq_biip_rotate",
                     "kronq_cholesky_inv", "kronq_quantize_layer", "kronq_pack", "kronq_unpack",
                     "kronq_layer_loss", "kronq_workspace_size", "kronq_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(L):
    for name in _declared():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_status_strings_and_version(L):
    assert L.kronq_status_string(0) == b"ok"
    assert L.kronq_status_string(-3) == b"matrix not positive definite"
    assert L.kronq_status_string(12345) == b"unknown status"
    assert L.kronq_abi_version() == 101


def test_sync_status_reports_the_stream(L):
    """kronq_sync_status waits for the stream: on a host without a usable
    device that wait itself fails and is reported as KRONQ_ERR_CUDA (-4),
    not raised; with a device and no work queued it is KRONQ_OK."""
    import torch
    expected = 0 if torch.cuda.is_available() else -4
    assert L.kronq_sync_status(None, None) == expected


def test_workspace_size(L):
    ws = L.kronq_workspace_size(4096, 4096, 4, -1, 128)
    # the inverse Cholesky needs two n x n fp32 scratch matrices
    assert ws >= 2 * 4096 * 4096 * 4
    assert L.kronq_launch_count() >= 0
    assert L.kronq_workspace_size(0, 4096, 4, -1, 128) == 0


def test_host_side_argument_errors(L):
    null = None
    # pack: 3-bit is not packable; bad widths invalid
    assert L.kronq_pack(null, 4, 16, 3, null, null) == -2
    assert L.kronq_pack(null, 4, 16, 5, null, null) == -1
    assert L.kronq_unpack(null, 4, 16, 3, null, null) == -2
    # empty inputs are a no-op
    assert L.kronq_pack(null, 0, 16, 4, null, null) == 0
    # quantize: group must divide n, block must be 128
    assert L.kronq_quantize_layer(null, 4, 256, null, 4, -1, 128, null, null, null, null, null,
                                  null, 0, null) == -1
    ptr = ctypes.c_void_p(16)  # never dereferenced: rejected before any launch
    assert L.kronq_quantize_layer(ptr, 4, 256, ptr, 4, 96, 128, ptr, ptr, ptr, null, null,
                                  null, 0, null) == -1
    assert L.kronq_quantize_layer(ptr, 4, 256, ptr, 4, -1, 64, ptr, ptr, ptr, null, null,
                                  null, 0, null) == -2
    assert L.kronq_quantize_layer(ptr, 4, 256, ptr, 5, -1, 128, ptr, ptr, ptr, null, null,
                                  null, 0, null) == -1
    # workspace too small
    assert L.kronq_quantize_layer(ptr, 4, 256, ptr, 4, -1, 128, ptr, ptr, ptr, null, null,
                                  null, 0, null) == -6
    # cholesky: aliasing and workspace
    assert L.kronq_cholesky_inv(ptr, 64, ctypes.c_float(0.01), ptr, null, null, 0, null) == -1
    assert L.kronq_cholesky_inv(ptr, 64, ctypes.c_float(0.01), ctypes.c_void_p(32), null, null,
                                0, null) == -6
    # biip: widths must be multiples of 16; an odd part above 63 is unsupported
    assert L.kronq_biip_rotate(ptr, 24, 64, ptr, ptr, ptr, ptr, ctypes.c_float(0.25), 0, 0, ptr,
                               ptr, null, 0, null) == -1
    assert L.kronq_biip_rotate(ptr, 16 * 65, 64, ptr, ptr, ptr, ptr, ctypes.c_float(0.25), 0, 0,
                               ptr, ptr, null, 0, null) == -2
    assert L.kronq_biip_rotate(ptr, 64, 64, ptr, ptr, ptr, ptr, ctypes.c_float(0.25), 7, 0, ptr,
                               ptr, null, 0, null) == -1
    # covariance: misaligned leading dimension, tiny width
    assert L.kronq_covariance(ptr, 10, 100, 100 + 3, ptr, 100, ctypes.c_float(1.0),
                              ctypes.c_float(0.0), null, null) == -1
    assert L.kronq_covariance(ptr, 10, 40, 40, ptr, 40, ctypes.c_float(1.0),
                              ctypes.c_float(0.0), null, null) == -2
    assert L.kronq_covariance(null, 10, 0, 0, null, 0, ctypes.c_float(1.0),
                              ctypes.c_float(0.0), null, null) == 0


def test_host_side_argument_errors_act_order_clip(L):
    null = None
    ptr = ctypes.c_void_p(16)  # never dereferenced: rejected before any launch
    # unknown option bits
    assert L.kronq_quantize_layer_opt(ptr, 4, 256, ptr, 4, -1, 128, 2, ptr, ptr, ptr, null, null,
                                      null, 0, null) == -1
    # the clip option passes the argument checks up to the workspace
    assert L.kronq_quantize_layer_opt(ptr, 4, 256, ptr, 4, -1, 128, 1, ptr, ptr, ptr, null, null,
                                      null, 0, null) == -6
    # act_order: empty is a no-op, null pointers invalid
    assert L.kronq_act_order(null, 0, null, null) == 0
    assert L.kronq_act_order(null, 8, ptr, null) == -1
    # permute: bad mode, aliasing, symmetric needs a square fp32 matrix, bad element size
    q = ctypes.c_void_p(32)
    assert L.kronq_permute(ptr, q, 4, 8, 4, ptr, 7, null, null) == -1
    assert L.kronq_permute(ptr, ptr, 4, 8, 4, ptr, 0, null, null) == -1
    assert L.kronq_permute(ptr, q, 4, 8, 4, ptr, 2, null, null) == -1
    assert L.kronq_permute(ptr, q, 8, 8, 1, ptr, 2, null, null) == -1
    assert L.kronq_permute(ptr, q, 4, 8, 2, ptr, 0, null, null) == -1
    assert L.kronq_permute(null, null, 0, 8, 4, null, 0, null, null) == 0


def test_host_side_argument_errors_deploy(L):
    null = None
    ptr = ctypes.c_void_p(256)  # never dereferenced: rejected before any launch
    args = lambda m, n, bits, group, mode, batch, ws_bytes: (
        ptr, m, n, bits, group, ptr, ptr, ptr, ptr, ptr, ptr, mode, ptr, batch, ptr, ptr, ws_bytes, null)
    assert L.kronq_deploy_matvec(null, 64, 128, 4, -1, ptr, ptr, ptr, ptr, ptr, ptr, 0, ptr, 1, ptr,
                                 ptr, 1 << 20, null) == -1          # null packed codes
    assert L.kronq_deploy_matvec(*args(64, 128, 3, -1, 0, 1, 1 << 20)) == -2   # 3-bit is not packed
    assert L.kronq_deploy_matvec(*args(64, 96, 4, -1, 0, 1, 1 << 20)) == -1    # n not a multiple of 64
    assert L.kronq_deploy_matvec(*args(64, 128, 4, 48, 0, 1, 1 << 20)) == -2   # group 48
    assert L.kronq_deploy_matvec(*args(64, 128, 4, -1, 5, 1, 1 << 20)) == -1   # unknown incoh mode
    assert L.kronq_deploy_matvec(*args(64, 128, 4, -1, 0, 3, 1 << 20)) == -2   # batch 3
    assert L.kronq_deploy_matvec(*args(64, 128, 4, -1, 0, 1, 0)) == -6         # workspace too small
    assert L.kronq_deploy_workspace_size(64, 128, 1) > 64 * 128
    assert L.kronq_deploy_workspace_size(0, 128, 1) == 0


def test_binding_refuses_host_tensors():
    import torch
    from post_quantization_02_b200 import abi
    with pytest.raises(ValueError):
        abi.kronq_covariance(torch.zeros(4, 64, dtype=torch.bfloat16),
                             torch.zeros(64, 64), 1.0)


def test_product_never_imports_the_oracle():
    pkg = ROOT / "post_quantization_02_b200"
    for f in list(pkg.glob("*.py")) + list((pkg / "csrc").glob("*")):
        text = f.read_text(errors="ignore")
        assert "oracle" not in re.findall(r"\b(?:import|from)\s+(\w+)", text), f


def _quant_tensors(m=8, n=256, G=1):
    import torch
    return dict(W=torch.zeros(m, n), U=torch.zeros(n, n),
                codes=torch.zeros(m, n, dtype=torch.uint8), scales=torch.zeros(m, G),
                zeros=torch.zeros(m, G, dtype=torch.uint8), W_hat=torch.zeros(m, n))


@pytest.mark.parametrize("bad", ["U", "codes", "scales", "zeros", "W_hat"])
@pytest.mark.parametrize("entry", ["kronq_quantize_layer", "kronq_quantize_layer_opt",
                                   "kronq_quantize_layer_noalloc"])
def test_binding_checks_solver_shapes(bad, entry):
    """Every solver tensor is checked against (m, n, G) before anything is
    passed on (a wrong shape would let the kernels run past its end)."""
    import torch
    from post_quantization_02_b200 import abi
    t = _quant_tensors(G=2)
    t[bad] = torch.zeros((3,) + tuple(t[bad].shape[1:]), dtype=t[bad].dtype)
    fn = getattr(abi, entry)
    extra = (0,) if entry.endswith("_opt") else ()
    with pytest.raises(ValueError, match="shape|elements"):
        fn(t["W"], t["U"], 4, 128, 128, *extra, t["codes"], t["scales"], t["zeros"], t["W_hat"])


def test_binding_checks_other_shapes():
    import torch
    from post_quantization_02_b200 import abi
    f32 = lambda *s: torch.zeros(*s)
    i8 = lambda n: torch.ones(n, dtype=torch.int8)
    with pytest.raises(ValueError, match="shape"):          # H_X must be n x n
        abi.kronq_biip_rotate(f32(8, 64), f32(32, 32), f32(8, 8), i8(8), i8(64), 0.25, "full", 0,
                              f32(64), f32(8), None)
    with pytest.raises(ValueError, match="elements"):       # sign_v has n entries
        abi.kronq_biip_rotate(f32(8, 64), f32(64, 64), f32(8, 8), i8(8), i8(32), 0.25, "full", 0,
                              f32(64), f32(8), None)
    with pytest.raises(ValueError, match="shape"):          # U_c must match H
        abi.kronq_cholesky_inv(f32(64, 64), 0.01, f32(32, 32), None, None)
    with pytest.raises(ValueError, match="shape"):          # H must be d x d
        abi.kronq_covariance(torch.zeros(4, 64, dtype=torch.bfloat16), f32(32, 32), 1.0)
    with pytest.raises(ValueError, match="shape"):          # packed words per row
        abi.kronq_pack(torch.zeros(4, 64, dtype=torch.uint8), 4, torch.zeros(4, 4, dtype=torch.int32))
    with pytest.raises(ValueError, match="shape"):          # W_hat matches W_ref
        abi.kronq_layer_loss(f32(8, 64), f32(8, 32), f32(64, 64), f32(8, 8),
                             torch.zeros(1, dtype=torch.float64), None)
    with pytest.raises(ValueError, match="elements"):       # perm has n entries
        abi.kronq_act_order(f32(64, 64), torch.zeros(32, dtype=torch.int32))


def test_binding_refuses_host_tensors_of_the_right_shape():
    from post_quantization_02_b200 import abi
    t = _quant_tensors()
    with pytest.raises(ValueError, match="CUDA"):
        abi.kronq_quantize_layer(t["W"], t["U"], 4, -1, 128, t["codes"], t["scales"], t["zeros"])


def test_sync_status_binding_checks_its_info_word():
    """The binding passes an int32 info word through and rejects any other
    dtype before calling the library."""
    import torch
    from post_quantization_02_b200 import abi
    with pytest.raises(ValueError):
        abi.kronq_sync_status(None, torch.zeros(1, dtype=torch.float32))
