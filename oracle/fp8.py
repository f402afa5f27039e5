"""FP8 E4M3 token rows of the mixed-format cache, float64.  Test
infrastructure only.

Minima-KV keeps recent and protected ("Anchor") pages in FP8 and older pages
in TQ3 ("KV-cache compresse et modeles 4-bit ...", section "Minima-KV : la
compression sans eviction").  The pages fix neither the FP8 variant nor its
scaling.  Readings:
* E4M3 as deployed on GPUs: 1 sign bit, 4 exponent bits with bias 7, 3
  mantissa bits, subnormals, no infinities, S.1111.111 is NaN, largest
  finite magnitude 448;
* one fp16 scale per token vector (key or value of one kv head):
  s = RNE_fp16(max_c |x_c| / 448), code_c = RNE_e4m3(x_c / s) (ties to even,
  magnitudes past 448 saturate to 448, which this scale never produces, and
  a value rounding to zero is coded +0), and x_hat_c = e4m3(code_c) * s;
  s = 0 (a zero vector) gives codes 0.
The quotients are taken in float64; max / 448 and x / s of 16-bit values are
never within float64 rounding of an fp16 or e4m3 midpoint without being on it,
so one rounding after the division decides exactly (pinned by a test against
exact rational rounding).
"""
from __future__ import annotations

import functools

import numpy as np

from .numerics import fp16_round

E4M3_MAX = 448.0


def e4m3_value(codes) -> np.ndarray:
    """Value of E4M3 bytes (float64; NaN for the NaN codes)."""
    c = np.asarray(codes, np.int64)
    s = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 15
    m = c & 7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return s * mag


@functools.lru_cache(maxsize=None)
def _positive_table():
    """The 127 finite non-negative E4M3 values, increasing with their codes."""
    return e4m3_value(np.arange(127))


def e4m3_encode(v) -> np.ndarray:
    """Nearest E4M3 code of float64 values, ties to the even code, magnitudes
    past 448 saturating to 448 (no NaN inputs)."""
    v = np.asarray(v, np.float64)
    tab = _positive_table()
    a = np.abs(v)
    i = np.clip(np.searchsorted(tab, a), 1, 126)            # tab[i-1] < a <= tab[i]
    lo, hi = tab[i - 1], tab[i]
    pick_hi = (a - lo > hi - a) | ((a - lo == hi - a) & (i % 2 == 0))
    code = np.where(pick_hi, i, i - 1)
    code = np.where(a >= E4M3_MAX, 126, code)
    code = np.where(a == 0.0, 0, code)
    # a value that rounds to zero is coded +0 (0x00) whatever its sign
    return (code | np.where((v < 0) & (code != 0), 128, 0)).astype(np.uint8)


def fp8_rows(x) -> tuple:
    """Token vectors x [T][d] (float64) -> (codes [T][d] uint8, scales [T]
    float64, each an fp16 value)."""
    x = np.asarray(x, np.float64)
    s = fp16_round(np.abs(x).max(axis=1) / E4M3_MAX)
    safe = np.where(s > 0, s, 1.0)
    codes = np.where(s[:, None] > 0, e4m3_encode(x / safe[:, None]), 0).astype(np.uint8)
    return codes, s


def fp8_dequant(codes, scales) -> np.ndarray:
    """x_hat [T][d] = e4m3(codes) * s."""
    return e4m3_value(codes) * np.asarray(scales, np.float64)[:, None]
