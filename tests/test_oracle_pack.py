"""Pins of the oracle's packing (hand-worked words, round trips)."""

import numpy as np
import pytest

from conftest import GOLDEN
from oracle import pack as P


def _fixture(name):
    lines = [l for l in (GOLDEN / name).read_text().splitlines() if not l.startswith("#")]
    codes = np.array(lines[0].split(), dtype=np.uint8)
    words = np.array([int(x, 16) for x in lines[1].split()], dtype=np.uint32)
    return codes, words


@pytest.mark.parametrize("name,bits", [("pack_4bit.txt", 4), ("pack_2bit.txt", 2)])
def test_pack_golden(name, bits):
    codes, words = _fixture(name)
    got = P.pack(codes[None, :], bits)
    np.testing.assert_array_equal(got[0], words)
    np.testing.assert_array_equal(P.unpack(got, len(codes), bits)[0], codes)


@pytest.mark.parametrize("bits", [2, 4])
def test_round_trip_every_code(bits):
    r = np.random.default_rng(bits)
    codes = r.integers(0, 2 ** bits, (9, 96), dtype=np.uint8)
    codes[0, :2 ** bits] = np.arange(2 ** bits)
    p = P.pack(codes, bits)
    assert p.shape == (9, 96 * bits // 32)
    np.testing.assert_array_equal(P.unpack(p, 96, bits), codes)


def test_three_bit_and_range_rejected():
    with pytest.raises(ValueError):
        P.words_per_row(16, 3)
    with pytest.raises(ValueError):
        P.pack(np.array([[4]], dtype=np.uint8), 2)
