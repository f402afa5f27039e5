"""Pins for the FP8 E4M3 part of the oracle against torch's independent
float8_e4m3fn conversion, exact rational rounding, and special inputs.  CPU
only."""
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import fp8
from oracle.numerics import fp16_round


def _torch_decode(codes):
    t = torch.tensor(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def test_decode_table_matches_torch():
    codes = np.arange(256)
    ours, theirs = fp8.e4m3_value(codes), _torch_decode(codes)
    assert np.array_equal(np.isnan(ours), np.isnan(theirs))
    ok = ~np.isnan(ours)
    assert np.array_equal(ours[ok], theirs[ok])
    assert np.nanmax(ours) == 448.0 and ours[1] == 2.0 ** -9        # largest and smallest positive


def test_encode_matches_torch_on_every_fp16_value_in_range():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    v = bits.view(np.float16).astype(np.float64)
    v = v[np.isfinite(v) & (np.abs(v) <= 448.0)]
    theirs = torch.tensor(v, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    theirs = np.where((theirs & 127) == 0, 0, theirs)                  # zero: +0 whatever the sign
    assert np.array_equal(fp8.e4m3_encode(v), theirs)


def _exact_nearest(q: Fraction) -> int:
    """Nearest E4M3 code to an exact rational (ties to the even code)."""
    tab = [Fraction(float(x)) for x in fp8.e4m3_value(np.arange(127))]
    a = abs(q)
    if a >= 448:
        c = 126
    else:
        c = min(range(127), key=lambda i: (abs(tab[i] - a), i % 2))
    return (c | 128) if (q < 0 and c != 0) else c


def test_quotient_decision_is_exact():
    rng = np.random.default_rng(0)
    for _ in range(3000):
        x = float(np.float16(rng.normal(0, 3)))
        s = float(fp16_round(abs(rng.normal(0, 0.02)) + 1e-4))
        assert int(fp8.e4m3_encode(x / s)) == _exact_nearest(Fraction(x) / Fraction(s))
    # exact midpoints between neighbours go to the even code
    for k in range(1, 120):
        a, b = fp8.e4m3_value(k), fp8.e4m3_value(k + 1)
        mid = (a + b) / 2
        assert int(fp8.e4m3_encode(mid)) == (k if k % 2 == 0 else k + 1)
        assert int(fp8.e4m3_encode(-mid)) == (k if k % 2 == 0 else k + 1) | 128


def test_rows_scale_round_trip_and_error_bound():
    rng = np.random.default_rng(1)
    # vectors already on the grid of their own scale come back exactly
    s = fp16_round(np.abs(rng.normal(0, 0.05, 20)) + 1e-3)
    codes = rng.integers(0, 255, (20, 64)).astype(np.uint8)
    codes[np.isnan(fp8.e4m3_value(codes))] = 0
    codes[:, 0] = 126                                                   # max |x| = 448 s pins the scale
    x = fp8.e4m3_value(codes) * s[:, None]
    c2, s2 = fp8.fp8_rows(x)
    assert np.array_equal(s2, s) and np.array_equal(fp8.e4m3_value(c2), fp8.e4m3_value(codes))
    # random vectors: |x - x_hat| <= half an E4M3 step (of |x|/s) times s
    x = rng.normal(0, 1, (50, 128)) * np.where(rng.random((50, 1)) < 0.2, 20.0, 1.0)
    c, s = fp8.fp8_rows(x)
    xh = fp8.fp8_dequant(c, s)
    a = np.abs(x) / s[:, None]
    step = np.where(a < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(a, 2.0 ** -6))) - 3))
    assert np.all(np.abs(x - xh) <= step / 2 * s[:, None] * (1 + 1e-12))
    assert np.all(np.abs(x).max(axis=1) / s <= 448.0 * (1 + 2.0 ** -10))


def test_zero_vector_has_zero_scale_and_codes():
    c, s = fp8.fp8_rows(np.zeros((2, 16)))
    assert np.all(c == 0) and np.all(s == 0)
    assert np.all(fp8.fp8_dequant(c, s) == 0)


# ------------------------------------------------------------------ mixed-format row
from oracle import mixed_cache, turbo                                   # noqa: E402
from oracle.numerics import decode16                                    # noqa: E402


def _mixed(d=128, R=64, A=64, seed=4):
    rng = np.random.default_rng(seed)
    pi = turbo.rotation(rng.standard_normal((d, d)))
    s = rng.standard_normal((128, d)).astype(np.float32).astype(np.float64)
    lv, th = turbo.deployed_codebook(d)
    return mixed_cache.MixedRow(d, R, A, "bf16", pi, s, lv, th), rng


def _bits(x):
    from quantized_kv_cache_18_b200.workloads import round_to_bf16_bits
    return round_to_bf16_bits(np.asarray(x, np.float32))


def test_mixed_row_without_tq3_is_plain_softmax_over_fp8_values():
    row, rng = _mixed()
    kb, vb = _bits(rng.normal(size=(100, 128))), _bits(rng.normal(size=(100, 128)))
    row.prefill(kb, vb)                                                  # 64 anchors + 36 window tokens
    assert row.tq == 0 and row.r == 36
    qb = _bits(rng.normal(size=(2, 128)))
    out = row.attention(qb, 0.1)
    k = fp8.fp8_dequant(*fp8.fp8_rows(decode16(kb, "bf16")))
    v = fp8.fp8_dequant(*fp8.fp8_rows(decode16(vb, "bf16")))
    q = decode16(qb, "bf16")
    for h in range(2):                                                   # textbook double loop
        sc = [0.1 * sum(q[h, c] * k[t, c] for c in range(128)) for t in range(100)]
        mx = max(sc)
        w = [np.exp(x - mx) for x in sc]
        ref = [sum(w[t] * v[t, c] for t in range(100)) / sum(w) for c in range(128)]
        assert np.allclose(out[h], ref, rtol=1e-12, atol=1e-12)


def test_mixed_row_bookkeeping_and_flush_from_fp8_values():
    row, rng = _mixed()
    S = 64 + 200
    kb, vb = _bits(rng.normal(size=(S, 128))), _bits(rng.normal(size=(S, 128)))
    row.prefill(kb, vb)
    assert row.tq == 128 and row.r == 72 and row.A + row.tq + row.r == S
    # after prefill the window holds the FP8 form of the last r input tokens
    c, s = fp8.fp8_rows(decode16(kb[-72:], "bf16"))
    assert np.array_equal(row.ring["k"][0][:72], c) and np.array_equal(row.ring["k"][1][:72], s)
    n_flush = 0
    for i in range(60):
        kn, vn = _bits(rng.normal(size=128)), _bits(rng.normal(size=128))
        before = row.tq
        row.append(kn, vn)
        if row.tq > before:
            n_flush += 1
            assert row.tq - before == 32 and row.r == 64
        assert 64 <= row.r < 96
    assert n_flush == 2 and row.A + row.tq + row.r == S + 60          # r: 72 -> 96 (flush) -> 96 (flush)
    # the anchors never change
    assert np.array_equal(row.anc["k"][0], fp8.fp8_rows(decode16(kb[:64], "bf16"))[0])


def test_mixed_row_attention_is_close_to_exact_attention():
    row, rng = _mixed()
    S = 64 + 400
    kb, vb = _bits(rng.normal(size=(S, 128))), _bits(rng.normal(size=(S, 128)))
    row.prefill(kb, vb)
    qb = _bits(rng.normal(size=(4, 128)))
    out = row.attention(qb, 1 / np.sqrt(128))
    k, v, q = decode16(kb, "bf16"), decode16(vb, "bf16"), decode16(qb, "bf16")
    sc = q @ k.T / np.sqrt(128)
    p = np.exp(sc - sc.max(axis=1, keepdims=True))
    ref = (p @ v) / p.sum(axis=1, keepdims=True)
    err_mixed = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    # the same tokens with every quantized token in TQ3 and the window exact:
    # FP8 anchors and an FP8 window must not do worse
    from oracle import turbo_cache
    tq_row = turbo_cache.TurboRow(128, 64, "bf16", row.Pi, row.S, row.levels, row.thresholds)
    tq_row.prefill(kb, vb)
    err_tq = np.linalg.norm(tq_row.attention(qb, 1 / np.sqrt(128)) - ref) / np.linalg.norm(ref)
    assert err_mixed < 0.3 and err_mixed <= 1.05 * err_tq


def test_fp8_row_format():
    c = np.arange(128, dtype=np.uint8)[None].repeat(2, 0)
    rows = mixed_cache.pack_fp8_rows(c, np.array([1.5, 0.0]))
    assert rows.shape == (2, 144)
    assert np.array_equal(rows[:, :128], c)
    assert rows[0, 128:130].view(np.float16)[0] == 1.5 and np.all(rows[:, 130:] == 0)
