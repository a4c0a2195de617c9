"""Parity of the deployment matvec (kronq_deploy_matvec) with the fp64
oracle (oracle/deploy.py): y = S_G^-1 U^T W_hat' V S_X^-1 x from packed
codes (KronQ README (GitHub), deploy path; KronQ summary (hyper.ai),
"Method", Eqs. 11-12), on seeded random layers: codes, grids, scales and
signs drawn on the host, so nothing the oracle sees comes from the GPU.

Tolerance: the GPU dequantizes exactly and accumulates in fp32 (a dot
product of n terms and two log2-depth transforms, each rounding at 2^-24
relative): 1e-5 relative Frobenius on y.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import rel_fro, t
from oracle import deploy as odep
from oracle import pack as opack
from post_quantization_02_b200 import abi

pytestmark = pytest.mark.gpu

TOL = 1e-5
MODES = ["full", "no_rescale", "su_only", "sv_only"]


def _layer(r, m, n, bits, group, mode):
    G = 1 if group == -1 else n // group
    codes = r.integers(0, 2 ** bits, (m, n)).astype(np.uint8)
    scales = r.uniform(0.005, 0.05, (m, G)).astype(np.float32)
    zeros = r.integers(0, 2 ** bits, (m, G)).astype(np.uint8)
    su = (1 - 2 * r.integers(0, 2, m)).astype(np.int8)
    sv = (1 - 2 * r.integers(0, 2, n)).astype(np.int8)
    in_s = mode in ("full", "sv_only")
    out_s = mode in ("full", "su_only")
    SX = (r.uniform(0.5, 2.0, n) if in_s else np.ones(n)).astype(np.float32)
    SG = (r.uniform(0.5, 2.0, m) if out_s else np.ones(m)).astype(np.float32)
    return codes, scales, zeros, su, sv, SX, SG


@pytest.mark.parametrize("m,n,bits,group,batch,mode", [
    (256, 256, 4, -1, 1, "full"), (256, 256, 2, 128, 2, "full"), (336, 448, 4, 32, 1, "full"),
    (448, 448, 2, 64, 4, "no_rescale"), (128, 1024, 4, 128, 8, "su_only"),
    (1024, 128, 2, -1, 1, "sv_only"), (4096, 4096, 4, -1, 1, "full"),
    (1024, 11008, 2, 128, 2, "full"),
    (64, 28672, 4, 64, 2, "full"),            # vectors beyond one CTA's shared memory: three launches
    (32, 28672, 2, -1, 1, "sv_only")])
def test_deploy_matvec_matches_oracle(cuda, m, n, bits, group, batch, mode):
    r = np.random.default_rng(m + 3 * n + bits + batch)
    codes, scales, zeros, su, sv, SX, SG = _layer(r, m, n, bits, group, mode)
    packed = opack.pack(codes, bits)
    x = r.standard_normal((batch, n)).astype(np.float32)
    y = torch.empty((batch, m), device=cuda)
    ws = abi.deploy_workspace(m, n, batch, cuda)
    abi.kronq_deploy_matvec(t(packed.view(np.int32), cuda), n, bits, group, t(scales, cuda),
                            t(zeros, cuda), t(SX, cuda), t(SG, cuda), t(su, cuda), t(sv, cuda), mode,
                            t(x, cuda), y, ws)
    ref = odep.deploy_matvec(packed, n, bits, group, scales, zeros, SX, SG, su, sv, x, mode)
    assert rel_fro(y.cpu().numpy(), ref) <= TOL, rel_fro(y.cpu().numpy(), ref)


def test_deploy_rejects_bad_shapes(cuda):
    r = np.random.default_rng(1)
    m, n = 64, 96                      # n not a multiple of 64
    codes, scales, zeros, su, sv, SX, SG = _layer(r, m, n, 4, -1, "full")
    packed = t(opack.pack(codes, 4).view(np.int32), cuda)
    x = torch.zeros((1, n), device=cuda)
    y = torch.empty((1, m), device=cuda)
    with pytest.raises(abi.KronqError):
        abi.kronq_deploy_matvec(packed, n, 4, -1, t(scales, cuda), t(zeros, cuda), t(SX, cuda),
                                t(SG, cuda), t(su, cuda), t(sv, cuda), "full", x, y,
                                abi.deploy_workspace(m, n, 1, cuda))
