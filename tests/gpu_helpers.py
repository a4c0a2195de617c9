"""Shared helpers for the -m gpu parity tests: seeded inputs on host and
device, and the comparison measures the tolerances are stated in."""

import numpy as np
import torch

import synth


def bf16_host(a32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits (the generator's rounding)."""
    return synth.f32_to_bf16_bits(a32)


def bf16_dev(bits: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)


def widen(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def spd(r: np.random.Generator, d: int, spread: float = 2.0, k: int | None = None) -> np.ndarray:
    k = k or 2 * d
    A = r.standard_normal((k, d)) * np.exp(r.uniform(-spread, spread, d))[None, :]
    return (A.T @ A / k).astype(np.float32)


def signs(r: np.random.Generator, d: int) -> np.ndarray:
    return (1 - 2 * r.integers(0, 2, d)).astype(np.int8)


def t(x, dev):
    return torch.from_numpy(np.ascontiguousarray(x)).to(dev)
