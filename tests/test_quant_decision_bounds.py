"""The 4-bit quantizer's decision rule, restated on the host in numpy.

The kernel decides a 4-bit code from an fp32 estimate r = fma(x, 1/s, -z/s):
k is r rounded half to even (adding and subtracting 1.5 * 2^23 in fp32), and
k stands when the unit is safe (z - min <= s/2 and max - z <= (L + 1/2) s)
and |r - k| < thr = 1/2 - 2^-22 (2L + 2 + |z/s|); every other code goes to
the exact comparison.  These tests check, over random units, units whose
zero-point is large against their scale, and values on the half-step grid
(exact ties), that every code the estimate decides equals the oracle's exact
decision, and that the estimate decides almost every code.  CPU only; the
arithmetic is restated here from the rule above, not taken from the kernel
sources."""
import zlib

import numpy as np
import pytest

from oracle import kivi
from oracle.numerics import fp16_round

F32 = np.float32
L4 = 15
K_ROUND = F32(12582912.0)            # 1.5 * 2^23
EB_UNIT = F32(2.384185791015625e-7)   # 2^-22


def _round16(x, dtype):
    """float64 values rounded to the 16-bit input format (nearest, ties even)."""
    x = np.asarray(x, np.float64)
    if dtype == "fp16":
        return fp16_round(x)
    b = x.astype(np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16 << 16   # round to nearest even on the upper 16 bits
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def _estimate(x, mn, mx):
    """(decided mask, estimated code) of 16-bit inputs x of units (mn, mx)."""
    s, z = kivi.params(mn, mx, 4)
    s32, z32 = s.astype(F32), z.astype(F32)
    with np.errstate(divide="ignore"):
        inv = np.where(s32 > 0, F32(1.0) / np.where(s32 > 0, s32, F32(1.0)), F32(0.0)).astype(F32)
    zinv = (z32 * inv).astype(F32)
    safe = (z - mn <= 0.5 * s) & (mx - z <= (L4 + 0.5) * s)
    thr = (F32(0.5) - EB_UNIT * ((F32(2.0 * L4) + F32(2.0)) + np.abs(zinv))).astype(F32)
    thr = np.where(safe, thr, F32(-1.0)).astype(F32)
    # x * inv is exact in float64 (24 + 24 significant bits); one float64 and
    # one fp32 rounding stand in for the fused multiply-add's single rounding
    r = (x * inv.astype(np.float64) - zinv.astype(np.float64)).astype(F32)
    k = ((r + K_ROUND).astype(F32) - K_ROUND).astype(F32)
    decided = np.abs((r - k).astype(F32)) < thr
    return decided, k.astype(np.int64), s, z


def _check(x, mn, mx, min_decided):
    decided, k, s, z = _estimate(x, mn, mx)
    exact = kivi.codes(x, s, z, 4)
    assert np.all(exact[decided] == k[decided]), "an estimate decided a code the exact rule does not give"
    assert np.all((k[decided] >= 0) & (k[decided] <= L4))
    assert decided.mean() >= min_decided, decided.mean()


def _units(rng, dtype, n_units, width, centre, spread):
    """n_units rows of `width` 16-bit inputs; each row is one unit."""
    c = centre + rng.normal(0.0, 1.0, (n_units, 1)) * abs(centre) * 0.1
    sc = spread * np.exp(rng.normal(0.0, 1.0, (n_units, 1)))
    x = _round16(c + sc * rng.normal(0.0, 1.0, (n_units, width)), dtype)
    return x, x.min(axis=1, keepdims=True), x.max(axis=1, keepdims=True)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("centre,spread", [(0.0, 1.0), (0.0, 1e-3), (3.0, 0.5), (-40.0, 8.0)])
def test_estimate_decides_like_the_exact_rule(dtype, centre, spread):
    rng = np.random.default_rng(zlib.crc32(f"{dtype} {centre} {spread}".encode()))
    x, mn, mx = _units(rng, dtype, 4000, 128, centre, spread)
    _check(x, mn, mx, 0.99)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_large_zero_points_against_the_scale(dtype):
    """|z| / s up to a few thousand: the estimate is least accurate there, and
    its margin widens with |z / s|.  Far from zero the 16-bit inputs are coarse
    (fp16 steps of 2 around 4000), so exact ties, which the estimate leaves to
    the exact rule, become common."""
    rng = np.random.default_rng(5)
    for off, floor in ((512.0, 0.95), (-300.0, 0.95), (1000.0, 0.9), (4000.0, 0.75)):
        x, mn, mx = _units(rng, dtype, 2000, 64, off, 1.5)
        _check(x, mn, mx, floor)


def test_exact_ties_go_to_the_exact_rule():
    """Inputs on the grid z + k s / 2 (z = 512, s = 1, fp16): the odd points are
    ties, which the estimate must leave to the exact rule (round half to
    even), and the even points it decides."""
    rng = np.random.default_rng(9)
    x = 512.0 + rng.integers(0, 2 * L4 + 1, (3000, 64)) / 2.0
    x[:, 0], x[:, 1] = 512.0, 512.0 + L4
    mn, mx = x.min(axis=1, keepdims=True), x.max(axis=1, keepdims=True)
    decided, k, s, z = _estimate(x, mn, mx)
    assert np.all(s == 1.0) and np.all(z == 512.0)
    tie = (x * 2) % 2 == 1
    assert not decided[tie].any()
    assert decided[~tie].all()
    _check(x, mn, mx, 0.45)


# ------------------------------------------------------------------ 2-bit thresholds
def _all_finite16(dtype):
    """Every finite value of the 16-bit format, ascending (each value once)."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    if dtype == "fp16":
        v = bits.astype(np.uint16).view(np.float16).astype(np.float64)
    else:
        with np.errstate(invalid="ignore"):   # the nan patterns
            v = (bits << 16).view(np.float32).astype(np.float64)
    return np.unique(v[np.isfinite(v)])


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_2bit_threshold_counts_give_the_exact_codes(dtype):
    """The 2-bit rule: with X_k = z + (k + 1/2) s (exact in float64), c_k is the
    smallest 16-bit value v with v >= X_k (v > X_k for even k, so that a tie
    goes to the even code), and the code of x is the number of c_k that x
    reaches.  Here c_k is found by searching the sorted set of all 16-bit
    values; for every 16-bit input of each unit the count must equal the
    oracle's exact round-half-even code."""
    vals = _all_finite16(dtype)
    rng = np.random.default_rng(17 if dtype == "fp16" else 18)
    checked = 0
    for _ in range(400):
        scale = float(np.exp(rng.uniform(np.log(1e-6), np.log(300.0))))
        lo, hi = np.sort(rng.normal(0.0, 1.0, 2)) * scale + rng.normal(0.0, 3.0) * scale
        lo_i = np.searchsorted(vals, lo)
        hi_i = max(np.searchsorted(vals, hi, side="right") - 1, lo_i)
        xs = vals[lo_i:hi_i + 1]
        mn, mx = xs[0], xs[-1]
        s, z = kivi.params(np.float64(mn), np.float64(mx), 2)
        if s == 0:
            continue
        count = np.zeros(xs.shape, np.int64)
        for k in range(3):
            X = z + (k + 0.5) * s
            i = np.searchsorted(vals, X, side="right" if k % 2 == 0 else "left")
            c = vals[i] if i < vals.size else np.inf
            count += xs >= c
        assert np.array_equal(count, kivi.codes(xs, s, z, 2)), (mn, mx, s, z)
        checked += xs.size
    assert checked > 100000
