"""Pins for the KIVI part of the oracle, against things other than the oracle
itself: exact rational arithmetic, closed forms, hand-worked positions of the
packed layout, the pages' worked numbers, and brute force.  CPU only."""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import attention as oatt
from oracle import kivi, layout, memory
from oracle.cache import KiviRow, quantized_len
from oracle.numerics import decode16, fp16_round

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append([f.strip() for f in line.split("|")])
    return rows


# ------------------------------------------------------------------ exact helpers
def _fp16_grid():
    """All finite positive fp16 values as Fractions, ascending."""
    bits = np.arange(0x0001, 0x7C00, dtype=np.uint16)
    return [Fraction(float(v)) for v in bits.view(np.float16).astype(np.float64)]


_GRID = None


def exact_fp16_round(x: Fraction) -> Fraction:
    """Nearest fp16 to a rational, ties to the even significand; inf past 65520."""
    global _GRID
    if _GRID is None:
        _GRID = _fp16_grid()
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    if a >= Fraction(65520):
        return sign * Fraction(10 ** 30)       # stands for inf
    import bisect
    i = bisect.bisect_left(_GRID, a)
    lo = _GRID[i - 1] if i > 0 else Fraction(0)
    hi = _GRID[i] if i < len(_GRID) else Fraction(65504)
    if a == hi:
        return sign * hi
    dlo, dhi = a - lo, hi - a
    if dlo < dhi:
        return sign * lo
    if dhi < dlo:
        return sign * hi
    # tie: the even significand has its last bit 0
    lo_bits = int(np.float16(float(lo)).view(np.uint16)) if lo != 0 else 0
    return sign * (lo if lo_bits % 2 == 0 else hi)


def exact_code(x: Fraction, s: Fraction, z: Fraction, bits: int) -> int:
    if s == 0:
        return 0
    r = (x - z) / s
    f = math.floor(r)
    frac = r - f
    q = f + (1 if frac > Fraction(1, 2) else 0)
    if frac == Fraction(1, 2):
        q = f if f % 2 == 0 else f + 1
    return int(min(max(q, 0), (1 << bits) - 1))


# ------------------------------------------------------------------ numerics
def test_fp16_round_matches_exact_rational_rounding():
    rng = np.random.default_rng(11)
    xs = list(rng.standard_normal(3000) * np.exp(rng.uniform(-12, 10, 3000)))
    # values at, just above and just below fp16 rounding midpoints
    grid = np.arange(0x0400, 0x7BFF, 37, dtype=np.uint16).view(np.float16).astype(np.float64)
    for g in grid:
        nxt = float(np.nextafter(np.float16(g), np.float16(np.inf)))
        mid = (g + nxt) / 2
        xs += [mid, np.nextafter(mid, np.inf), np.nextafter(mid, -np.inf)]
    got = fp16_round(np.array(xs))
    for x, y in zip(xs, got):
        assert Fraction(float(y)) == exact_fp16_round(Fraction(float(x))), x


def test_scale_double_rounding_is_harmless():
    """s = fp16(float64((mx - mn) / (2^b - 1))) equals the fp16 rounding of the
    exact quotient for 16-bit mx, mn (random sample of fp16 and bf16 pairs)."""
    rng = np.random.default_rng(5)
    for bits in (2, 4):
        levels = (1 << bits) - 1
        a = rng.standard_normal(4000) * np.exp(rng.uniform(-6, 8, 4000))
        b = a + np.abs(rng.standard_normal(4000)) * np.exp(rng.uniform(-6, 8, 4000))
        for dt in ("fp16", "bf16"):
            if dt == "fp16":
                mn, mx = fp16_round(a), fp16_round(b)
            else:
                mn = a.astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
                mx = b.astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
                mn, mx = mn.view(np.float32).astype(np.float64), mx.view(np.float32).astype(np.float64)
            ok = np.isfinite(mn) & np.isfinite(mx) & (mx >= mn)
            s, _ = kivi.params(mn[ok], mx[ok], bits)
            for lo, hi, got in zip(mn[ok][:1500], mx[ok][:1500], s[:1500]):
                want = exact_fp16_round((Fraction(float(hi)) - Fraction(float(lo))) / levels)
                if want > 65504:
                    assert np.isinf(got)
                else:
                    assert Fraction(float(got)) == want


def test_codes_match_exact_rounding_including_ties():
    rng = np.random.default_rng(7)
    for bits in (2, 4):
        levels = (1 << bits) - 1
        for _ in range(60):
            vals = fp16_round(rng.standard_normal(40) * rng.uniform(0.1, 30))
            s, z = kivi.params(vals.min(), vals.max(), bits)
            # plant exact ties z + (k + 1/2) s when representable, and grid points
            extra = []
            for k in range(levels):
                for cand in (z + (k + 0.5) * s, z + k * s):
                    if fp16_round(cand) == cand and vals.min() <= cand <= vals.max():
                        extra.append(cand)
            x = np.concatenate([vals, np.array(extra)])
            got = kivi.codes(x, s, z, bits)
            for xi, gi in zip(x, got):
                assert gi == exact_code(Fraction(float(xi)), Fraction(float(s)), Fraction(float(z)), bits)


def test_tie_rule_is_half_to_even():
    s, z = 1.0, 0.0
    x = np.array([0.5, 1.5, 2.5, 3.5, 0.49, 0.51])
    assert kivi.codes(x, s, z, 2).tolist() == [0, 2, 2, 3, 0, 1]


def test_code_decision_is_exact_when_float64_subtraction_rounds():
    """x - z inexact in float64 (|z| >> |x|): the error-free sum keeps the
    comparison exact."""
    z = -100.0
    s = 40.0                         # thresholds 40, 120, 200 in units of 2(x - z)
    x = 2.0 ** -60                   # 2(x - z) = 200 + 2^-59 > 200: code 3
    assert kivi.codes(np.array([x]), s, z, 2)[0] == 3
    assert kivi.codes(np.array([0.0]), s, z, 2)[0] == 2    # exact tie at k = 2: even


# ------------------------------------------------------------------ quantizer properties
def _rand_groups(rng, n, G, d, dtype):
    x = rng.standard_normal((n, G, d)).astype(np.float32)
    x[:, :, :3] *= 20
    if dtype == "fp16":
        bits = x.astype(np.float16).view(np.uint16)
    else:
        u = x.view(np.uint32)
        bits = ((u + (((u >> 16) & 1) + 0x7FFF)) >> 16).astype(np.uint16)
    return decode16(bits, dtype)


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_error_bound(bits, dtype):
    """|x - x_hat| <= s/2 for every element not clamped; clamped elements stay
    within s/2 + (2^b-1)|s - s_exact| + |min - z|."""
    rng = np.random.default_rng(3)
    levels = (1 << bits) - 1
    for g in _rand_groups(rng, 30, 32, 16, dtype):
        c, s, z = kivi.quantize_keys(g, bits)
        xh = kivi.dequant(c, s[None], z[None])
        err = np.abs(g - xh)
        s_exact = (g.max(0) - g.min(0)) / levels
        interior = (c > 0) & (c < levels)
        assert np.all(err[interior] <= s[None].repeat(32, 0)[interior] / 2)
        bound = s / 2 + levels * np.abs(s - s_exact) + np.abs(g.min(0) - z)
        assert np.all(err <= bound[None] * (1 + 1e-12))


def test_error_bound_shrinks_with_bits():
    rng = np.random.default_rng(4)
    g = _rand_groups(rng, 1, 64, 32, "fp16")[0]
    errs = []
    for b in range(2, 9):
        c, s, z = kivi.quantize_keys(g, b)
        errs.append(np.abs(g - kivi.dequant(c, s[None], z[None])).max())
    rng_ = (g.max(0) - g.min(0)).max()
    for b, e in zip(range(2, 9), errs):
        assert e <= rng_ / (2 * ((1 << b) - 1)) * 1.01 + 1e-3
    assert all(errs[i + 1] < errs[i] for i in range(len(errs) - 1))


@pytest.mark.parametrize("bits", [2, 4])
def test_grid_round_trip(bits):
    """x = z + k s quantize to k and dequantize to x exactly."""
    levels = (1 << bits) - 1
    rng = np.random.default_rng(9)
    for _ in range(50):
        z = fp16_round(rng.standard_normal() * 10)
        s = fp16_round(abs(rng.standard_normal()) + 0.01)
        k = rng.integers(0, levels + 1, 64)
        k[0], k[1] = 0, levels            # the group spans the full grid
        x = z + k * s
        if not np.all(fp16_round(x) == x):
            continue
        c, s2, z2 = kivi.quantize_keys(np.repeat(x[:, None], 3, axis=1), bits)
        assert np.all(s2 == s) and np.all(z2 == z)
        assert np.array_equal(c[:, 0], k)
        assert np.array_equal(kivi.dequant(c, s2[None], z2[None])[:, 0], x)


def test_constant_group_gives_zero_codes():
    g = np.full((32, 8), 3.25)
    c, s, z = kivi.quantize_keys(g, 2)
    assert np.all(c == 0) and np.all(s == 0) and np.all(z == 3.25)
    assert np.array_equal(kivi.dequant(c, s[None], z[None]), g)


def test_group_batch_equals_single_groups():
    rng = np.random.default_rng(12)
    k = _rand_groups(rng, 5, 32, 16, "bf16").reshape(160, 16)
    c, s, z = kivi.quantize_key_groups(k, 2, 32)
    for i in range(5):
        c1, s1, z1 = kivi.quantize_keys(k[32 * i:32 * (i + 1)], 2)
        assert np.array_equal(c[32 * i:32 * (i + 1)], c1) and np.array_equal(s[i], s1) and np.array_equal(z[i], z1)


def test_keys_per_channel_values_per_token():
    """Channel outliers blow up a per-token scale but not a per-channel one, and
    token outliers the reverse: the reason the pages give for the K/V split."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((32, 64))
    xk = x.copy(); xk[:, 5] *= 50          # key-like: one outlier channel
    xv = x.copy(); xv[7, :] *= 50          # value-like: one outlier token
    ck, sk, zk = kivi.quantize_keys(xk, 2)
    cv, sv, zv = kivi.quantize_values(xv, 2)
    err_k_chan = np.abs(xk - kivi.dequant(ck, sk[None], zk[None]))[:, np.arange(64) != 5].max()
    c2, s2, z2 = kivi.quantize_values(xk, 2)
    err_k_tok = np.abs(xk - kivi.dequant(c2, s2[:, None], z2[:, None]))[:, np.arange(64) != 5].max()
    assert err_k_chan < err_k_tok / 5
    err_v_tok = np.abs(xv - kivi.dequant(cv, sv[:, None], zv[:, None]))[np.arange(32) != 7].max()
    c3, s3, z3 = kivi.quantize_keys(xv, 2)
    err_v_chan = np.abs(xv - kivi.dequant(c3, s3[None], z3[None]))[np.arange(32) != 7].max()
    assert err_v_tok < err_v_chan / 5


# ------------------------------------------------------------------ layout
def test_layout_density_matches_pages():
    for bits, per_word, reduction in [(int(a), int(b), int(c)) for a, b, c in _golden("packing_ratios.txt")]:
        assert 32 // bits == per_word
        assert memory.codes_only_ratio(bits) == reduction
        for d in (64, 128):
            off, bit = layout.key_code_map(d, bits)
            # every 32-bit word of a TB holds exactly 32/bits codes
            words = off // 4
            assert np.all(np.bincount(words.ravel()) == per_word)
            assert layout.tb_code_bytes(d, bits) == 32 * d * bits // 8


def test_layout_hand_worked_positions():
    """Positions worked by hand from the format table (d = 128, 2-bit).
    Key: token 9, channel 3 -> nt 1, gr 1, kt 0, rho 0, tc 1, e 1 -> lane 5;
    u 0 -> j' 0, slot 4, word 2, j 0 -> bit 16, byte 16*5 + 4*2 = 88.
    Value: token 9, channel 3 -> kt 0, rho 1, tc 0, e 1, nt 0, gr 3 -> lane 12;
    u 1 -> j' 1, slot 0, word 0, j 1 -> bit 2 + 16 = 18, byte 16*12 = 192."""
    off, bit = layout.key_code_map(128, 2)
    assert (off[9, 3], bit[9, 3]) == (88, 16)
    off, bit = layout.value_code_map(128, 2)
    assert (off[9, 3], bit[9, 3]) == (192, 18)
    # 4-bit key: token 0, channel 40 -> nt 0, gr 0, kt 2, rho 1, tc 0, e 0, lane 0;
    # u 5 -> j' 1, slot 2, word 1, j 1 -> bit 4, byte 4
    off, bit = layout.key_code_map(128, 4)
    assert (off[0, 40], bit[0, 40]) == (4, 4)
    # key meta: channel 19 = 16*1 + 0 + 2*1 + 1 -> kt 1, rho 0, tc 1, e 1
    #   -> 8*(4*0 + 1) + 4*1 + 0 + 1 = 13
    assert layout.key_meta_perm(128)[19] == 13
    # channel 125 = 16*7 + 8 + 2*2 + 1 -> kt 7, rho 1, tc 2, e 1 -> 8*(12 + 2) + 4 + 2 + 1 = 119
    assert layout.key_meta_perm(128)[125] == 119
    # value meta: token 27 = 16 + 8 + 2*1 + 1 -> tc 1 -> 8 + 4 + 2 + 1 = 15
    assert layout.value_meta_perm()[27] == 15


@pytest.mark.parametrize("d,bits,G", [(64, 2, 32), (128, 2, 32), (128, 4, 64)])
def test_layout_round_trip(d, bits, G):
    rng = np.random.default_rng(d + bits)
    T = 3 * G
    kc = rng.integers(0, 1 << bits, (T, d)).astype(np.uint8)
    vc = rng.integers(0, 1 << bits, (T, d)).astype(np.uint8)
    ks = fp16_round(rng.uniform(0, 3, (T // G, d)))
    kz = fp16_round(rng.standard_normal((T // G, d)))
    vs = fp16_round(rng.uniform(0, 3, T))
    vz = fp16_round(rng.standard_normal(T))
    rec = layout.pack_records(kc, ks, kz, vc, vs, vz, d, bits, G)
    assert rec.shape == (T // G, layout.record_bytes(d, bits, G))
    out = layout.unpack_records(rec, d, bits, G)
    for a, b in zip(out, (kc, ks, kz, vc, vs, vz)):
        assert np.array_equal(a, b)


def test_record_sizes():
    assert layout.record_bytes(128, 2, 32) == 2688
    assert layout.record_bytes(128, 4, 64) == 8960
    assert layout.record_bytes(64, 2, 32) == 1408
    # per token and head: 84 B (2-bit G32), 140 B (4-bit G64), 44 B (tiny)
    assert memory.kivi_bytes_per_token(128, 2, 32) == 84
    assert memory.kivi_bytes_per_token(128, 4, 64) == 140
    assert memory.kivi_bytes_per_token(64, 2, 32) == 44


# ------------------------------------------------------------------ memory formula
def test_memory_formula_matches_page_numbers():
    g = {r[0]: float(r[1]) for r in _golden("memory_formula.txt")}
    per_token = memory.kv_cache_bytes(80, 8, 128, 1, 2)
    assert per_token == 327680
    assert abs(per_token / 2 ** 20 - g["llama31_70b_bytes_per_token"]) < 0.005
    t128 = memory.kv_cache_bytes(80, 8, 128, 131072, 2)
    assert round(t128 / 2 ** 30) == g["llama31_70b_128k_total"]
    assert math.floor(t128 / 1e9) == g["llama31_70b_128k_total_alt"]
    assert memory.kv_cache_bytes(80, 8, 128, 2 ** 20, 2) / 1e9 > g["llama31_70b_1m_total_lower_bound"]


def test_minima_kv_byte_consistency():
    g = {r[0]: float(r[1]) for r in _golden("minima_kv.txt")}
    bf16 = g["kib_per_token"] * g["ratio_vs_bf16"]
    fp8 = g["kib_per_token"] * g["ratio_vs_fp8"]
    assert abs(bf16 / fp8 - 2.0) < 1e-9
    # bf16 bytes per token of the formula with L*H*d = 16384 gives the same 64 KiB
    assert abs(memory.kv_cache_bytes(1, 1, 16384, 1, 2) / 1024 - bf16) < 0.1


def test_workload_packed_bytes():
    """Bytes one decode step reads on the five workloads (window included)."""
    cases = [  # B, Hkv, d, bits, G, S, R
        (1, 2, 64, 2, 32, 512, 32, 58624),
        (16, 8, 128, 2, 32, 8192, 128, 95092736),
        (64, 8, 128, 4, 64, 4096, 128, 317980672),
        (1, 8, 128, 2, 32, 131072, 128, 88518656),
    ]
    for B, H, d, bits, G, S, R, want in cases:
        tq = quantized_len(S, R, G)
        assert memory.kivi_cache_bytes(B, H, d, bits, G, tq, S - tq) == want


# ------------------------------------------------------------------ window bookkeeping
def _scratch_state(tokens_k, tokens_v, S0, R, G, bits, d):
    """Closed-form model: the quantized length after a prefill of S0 and n
    appends, then every quantized group re-quantized from scratch."""
    n = len(tokens_k) - S0
    tq0 = quantized_len(S0, R, G)
    r0 = S0 - tq0
    flushes = max(0, (r0 + n - R) // G) if r0 + n >= R + G else 0
    tq = tq0 + G * flushes
    k = decode16(np.array(tokens_k), "fp16")
    v = decode16(np.array(tokens_v), "fp16")
    kc = [kivi.quantize_keys(k[i:i + G], bits) for i in range(0, tq, G)]
    vcs = kivi.quantize_values(v[:tq], bits) if tq else None
    return tq, kc, vcs


@pytest.mark.parametrize("G,R,steps", [(4, 4, 12), (4, 8, 12), (32, 32, 70)])
def test_window_bookkeeping_brute_force(G, R, steps):
    """Every prefill length up to 40 (and the boundary lengths) followed by
    every append count up to `steps`, on d = 8 (the row model does not depend
    on d): incremental state == closed-form quantized length + groups
    re-quantized from scratch, window == the last r tokens."""
    d, bits = 8, 2
    rng = np.random.default_rng(0)
    for S0 in sorted(set(list(range(0, 41)) + [R - 1, R, R + G - 1, R + G, 2 * R + G + 5])):
        total = S0 + steps
        kb = rng.standard_normal((total, d)).astype(np.float16).view(np.uint16)
        vb = rng.standard_normal((total, d)).astype(np.float16).view(np.uint16)
        row = KiviRow(d, bits, G, R, "fp16")
        row.prefill(kb[:S0], vb[:S0])
        for n in range(0, steps + 1):
            if n:
                row.append(kb[S0 + n - 1], vb[S0 + n - 1])
            S = S0 + n
            assert row.seq_len == S
            assert row.tq % G == 0
            if S >= R:
                assert R <= row.r < R + G
            tq, kc, vcs = _scratch_state(list(kb[:S]), list(vb[:S]), S0, R, G, bits, d)
            assert row.tq == tq
            for gi, (c, s, z) in enumerate(kc):
                assert np.array_equal(row.kc[gi * G:(gi + 1) * G], c)
                assert np.array_equal(row.ks[gi], s) and np.array_equal(row.kz[gi], z)
            if tq:
                assert np.array_equal(row.vc, vcs[0]) and np.array_equal(row.vs, vcs[1])
            wk, wv = row.window_bits()
            assert np.array_equal(wk, kb[tq:S]) and np.array_equal(wv, vb[tq:S])


# ------------------------------------------------------------------ attention
def test_attention_without_quantized_tokens_is_plain_softmax():
    """R >= S: nothing is quantized and the row attention is textbook softmax
    attention over the exact inputs."""
    rng = np.random.default_rng(2)
    d, S = 16, 20
    kb = rng.standard_normal((S, d)).astype(np.float16).view(np.uint16)
    vb = rng.standard_normal((S, d)).astype(np.float16).view(np.uint16)
    row = KiviRow(d, 2, 32, 32, "fp16")
    row.prefill(kb, vb)
    assert row.tq == 0
    K, V = row.dequantized()
    q = rng.standard_normal((3, d))
    got = oatt.attention(q, K, V, 0.25)
    want = np.array(oatt.attention_loops(q.tolist(), decode16(kb, "fp16").tolist(),
                                         decode16(vb, "fp16").tolist(), 0.25))
    assert np.abs(got - want).max() < 1e-12


def test_split_merge_invariance():
    rng = np.random.default_rng(8)
    q = rng.standard_normal((4, 32))
    K = rng.standard_normal((300, 32)) * 3
    V = rng.standard_normal((300, 32))
    full = oatt.attention(q, K, V, 0.2)
    for cuts in ([0, 300], [0, 1, 300], [0, 17, 100, 101, 299, 300], list(range(0, 301, 30))):
        parts = [oatt.partial(q, K[a:b], V[a:b], 0.2) for a, b in zip(cuts[:-1], cuts[1:])]
        assert np.abs(oatt.merge(parts) - full).max() < 1e-12


def test_single_token_attention_returns_its_value():
    q = np.ones((2, 4))
    K = np.zeros((1, 4))
    V = np.array([[1.0, -2.0, 3.0, 0.5]])
    assert np.array_equal(oatt.attention(q, K, V, 1.0), np.repeat(V, 2, axis=0))
