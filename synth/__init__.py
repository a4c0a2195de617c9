"""Seeded synthetic inputs for the KronQ layer-quantization path.

This package draws random numbers and nothing else: weights W, calibration
activations X, output gradients G and the random sign vectors of the two
Hadamard rotations.  It holds none of the method's arithmetic (no covariance,
no rotation, no quantizer), so the fp64 oracle and the CUDA path can both be
fed from it without sharing any code of the method.

Every stream is a Philox counter-based generator keyed by
(seed, tensor id, sublayer or site index, token chunk), so any token range of
X or G can be regenerated on its own, in any order, by either side.
"""

from .configs import CONFIGS, Config, Sublayer, XSite, get_config
from .gen import (
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    make_g,
    make_signs,
    make_w,
    make_x,
    make_xq,
    g_chunk,
    x_chunk,
    xq_chunk,
    n_chunks,
    CHUNK_TOKENS,
)

__all__ = [
    "CONFIGS", "Config", "Sublayer", "XSite", "get_config",
    "bf16_bits_to_f32", "f32_to_bf16_bits", "make_g", "make_signs", "make_w",
    "make_x", "make_xq", "g_chunk", "x_chunk", "xq_chunk", "n_chunks", "CHUNK_TOKENS",
]
