"""KIVI-style asymmetric quantizer, float64.  Test infrastructure only.

What the pages fix (zubnet.ai survey, "Famille deux, c'est la quantification";
"Quantification du KV-Cache : TurboQuant et l'etat de l'art en 2026", section
"KIVI (2024) -- la quantification asymetrique par canal"): keys are quantized
per channel and values per token, each with its own min/max parameters, at
2 bits (the 4-bit width follows the same recipe), with the most recent tokens
kept unquantized.

Readings where the pages are silent:
* asymmetric parameters: s = (max - min) / (2^b - 1) rounded to fp16 (ties to
  even), z = min rounded to fp16;
* code = clamp(round_half_even((x - z) / s), 0, 2^b - 1), decided exactly by
  comparing 2(x - z) with (2k + 1) s; s == 0 gives code 0;
* dequantized value x_hat = z + code * s;
* key groups are G consecutive tokens per channel; a value "group" is one token
  across all d channels.
"""
from __future__ import annotations

import numpy as np

from .numerics import fp16_round, two_sum


def params(mn: np.ndarray, mx: np.ndarray, bits: int):
    """(scale, zero) as float64 values of fp16 numbers.

    (mx - mn) is exact in float64 for 16-bit inputs; the quotient is rounded
    once to float64 and then to fp16."""
    levels = (1 << bits) - 1
    s = fp16_round((np.asarray(mx, np.float64) - np.asarray(mn, np.float64)) / levels)
    z = fp16_round(mn)
    return s, z


def codes(x: np.ndarray, s: np.ndarray, z: np.ndarray, bits: int) -> np.ndarray:
    """Round-half-even codes of x on the grid z + k s, k in [0, 2^b - 1].

    t = 2(x - z) is carried exactly as hi + lo (error-free sum); each threshold
    (2k + 1) s has at most 16 significant bits and is exact in float64, so every
    comparison below is exact.  Broadcasting: x, s and z broadcast together."""
    x = np.asarray(x, np.float64)
    s = np.asarray(s, np.float64)
    z = np.asarray(z, np.float64)
    hi, lo = two_sum(x, -z)
    t_hi, t_lo = 2.0 * hi, 2.0 * lo
    q = np.zeros(np.broadcast(x, s, z).shape, dtype=np.int64)
    for k in range((1 << bits) - 1):
        T = (2 * k + 1) * s
        above = (t_hi > T) | ((t_hi == T) & (t_lo > 0))
        tie = (t_hi == T) & (t_lo == 0)
        q += above.astype(np.int64)
        if k % 2 == 1:               # halfway between odd k and even k + 1: take k + 1
            q += tie.astype(np.int64)
    q[np.broadcast_to(s == 0, q.shape)] = 0
    return q.astype(np.uint8)


def in_range(x: np.ndarray, s: np.ndarray, z: np.ndarray) -> bool:
    """False when an input is non-finite or a parameter overflowed fp16 (the codes
    are then unspecified and the device status word flags the row)."""
    return bool(np.all(np.isfinite(x)) and np.all(np.isfinite(s)) and np.all(np.isfinite(z)))


def quantize_keys(kg: np.ndarray, bits: int):
    """One key group [G][d] -> (codes [G][d], scale [d], zero [d]): per channel."""
    kg = np.asarray(kg, np.float64)
    s, z = params(kg.min(axis=0), kg.max(axis=0), bits)
    return codes(kg, s[None, :], z[None, :], bits), s, z


def quantize_key_groups(k: np.ndarray, bits: int, G: int):
    """Consecutive key groups [n*G][d] -> (codes [n*G][d], scale [n][d],
    zero [n][d]); the same per-channel arithmetic as quantize_keys, for every
    group at once."""
    k = np.asarray(k, np.float64)
    n, d = k.shape[0] // G, k.shape[1]
    kg = k.reshape(n, G, d)
    s, z = params(kg.min(axis=1), kg.max(axis=1), bits)
    return codes(kg, s[:, None, :], z[:, None, :], bits).reshape(n * G, d), s, z


def quantize_values(v: np.ndarray, bits: int):
    """Value tokens [T][d] -> (codes [T][d], scale [T], zero [T]): per token."""
    v = np.asarray(v, np.float64)
    s, z = params(v.min(axis=1), v.max(axis=1), bits)
    return codes(v, s[:, None], z[:, None], bits), s, z


def dequant(c: np.ndarray, s: np.ndarray, z: np.ndarray) -> np.ndarray:
    return np.asarray(z, np.float64) + c.astype(np.float64) * np.asarray(s, np.float64)
