"""Packing of integer codes into 32-bit words.

KronQ README (GitHub), intro and "Model zoo": W4 and W2 are stored as real
packed int4 / int2; 3-bit is not bit-packable and ships as fake-quant.

Reading of the bit order (the pages do not give it): along each row, code
(i, j) goes to word (i, floor(j b / 32)), bits [(j mod 32/b) b, +b), so the
lowest-index code sits in the least significant bits.  A row of n codes
takes ceil(n b / 32) words; unused high bits of the last word are zero.
"""

from __future__ import annotations

import numpy as np


def words_per_row(n: int, bits: int) -> int:
    if bits not in (2, 4):
        raise ValueError("only 2- and 4-bit codes are packed")
    per = 32 // bits
    return (n + per - 1) // per


def pack(codes: np.ndarray, bits: int) -> np.ndarray:
    codes = np.asarray(codes)
    m, n = codes.shape
    per = 32 // bits
    nw = words_per_row(n, bits)
    out = np.zeros((m, nw), dtype=np.uint64)
    mask = (1 << bits) - 1
    if codes.size and int(codes.max()) > mask:
        raise ValueError("code out of range for the bit width")
    for j in range(n):
        out[:, j // per] |= (codes[:, j].astype(np.uint64) & np.uint64(mask)) << np.uint64((j % per) * bits)
    return out.astype(np.uint32)


def unpack(packed: np.ndarray, n: int, bits: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint64)
    m = packed.shape[0]
    per = 32 // bits
    mask = np.uint64((1 << bits) - 1)
    out = np.zeros((m, n), dtype=np.uint8)
    for j in range(n):
        out[:, j] = ((packed[:, j // per] >> np.uint64((j % per) * bits)) & mask).astype(np.uint8)
    return out
