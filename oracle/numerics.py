"""Number formats used by the oracle: 16-bit input decoding and fp16 rounding.

Test infrastructure only (see the package docstring).
"""
from __future__ import annotations

import numpy as np


def decode16(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of 16-bit patterns (bf16 or fp16)."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == "bf16":
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    if dtype == "fp16":
        return bits.view(np.float16).astype(np.float64)
    raise ValueError(dtype)


def fp16_round(x) -> np.ndarray:
    """Round float64 values to the nearest fp16 value (ties to even), returned as
    float64.  Overflow gives +-inf.  numpy converts float64 -> float16 directly
    (one rounding); a test pins this against exact rational rounding."""
    with np.errstate(over="ignore"):
        return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def fp16_bits(x) -> np.ndarray:
    """fp16 bit patterns of values that are already fp16-representable."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def two_sum(a: np.ndarray, b: np.ndarray):
    """Knuth's error-free sum: a + b == hi + lo exactly (no overflow)."""
    hi = a + b
    bb = hi - a
    lo = (a - (hi - bb)) + (b - bb)
    return hi, lo
