"""Pins for the TurboQuant part of the oracle against things other than the
oracle itself: the published Max (1960) table, numerical integration,
Gram-Schmidt, Monte Carlo over random sketches, special inputs, and
hand-worked layout positions.  CPU only."""
import math
import os

import numpy as np
import pytest
from scipy import integrate

from oracle import turbo, turbo_cache
from oracle.numerics import decode16, fp16_round

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = [f.strip() for f in line.split("|")]
            out[k] = [float(x) for x in v.split()]
    return out


# ------------------------------------------------------------------ Lloyd-Max
def test_lloyd_max_matches_max_1960_table():
    g = _golden("lloyd_max_gaussian8.txt")
    c, t = turbo.lloyd_max_gaussian(8)
    assert np.allclose(c[4:], g["levels"], atol=6e-4)
    assert np.allclose(-c[:4][::-1], g["levels"], atol=6e-4)
    assert np.allclose(t[3:], g["thresholds"], atol=6e-4)
    assert abs(turbo.gaussian_mse(c, t) - g["mse"][0]) < 2e-5


def test_lloyd_max_is_a_fixed_point_by_integration():
    """Each level is the conditional mean of its cell, computed here by
    adaptive quadrature (an independent routine)."""
    c, t = turbo.lloyd_max_gaussian(8)
    phi = lambda x: math.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)
    edges = [-np.inf] + list(t) + [np.inf]
    for k in range(8):
        a, b = edges[k], edges[k + 1]
        mass = integrate.quad(phi, a, b, epsabs=1e-14, epsrel=1e-13)[0]
        first = integrate.quad(lambda x: x * phi(x), a, b, epsabs=1e-14, epsrel=1e-13)[0]
        assert abs(first / mass - c[k]) < 1e-9
    assert np.allclose(t, 0.5 * (c[1:] + c[:-1]))


def test_mse_closed_form_matches_quadrature():
    c, t = turbo.lloyd_max_gaussian(8)
    phi = lambda x: math.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)
    edges = [-np.inf] + list(t) + [np.inf]
    mse = sum(integrate.quad(lambda x, k=k: (x - c[k]) ** 2 * phi(x), edges[k], edges[k + 1])[0] for k in range(8))
    assert abs(mse - turbo.gaussian_mse(c, t)) < 1e-9


def test_deployed_codebook_is_fp16_and_symmetric():
    lv, th = turbo.deployed_codebook(128)
    assert np.array_equal(fp16_round(lv), lv)
    assert np.array_equal(lv, -lv[::-1])
    assert th[3] == 0.0 and np.all(np.diff(lv) > 0)
    c, _ = turbo.lloyd_max_gaussian(8)
    assert np.allclose(lv, c / math.sqrt(128), rtol=1e-3)


# ------------------------------------------------------------------ rotation
def _gram_schmidt(a):
    q = np.zeros_like(a)
    for j in range(a.shape[1]):
        v = a[:, j].copy()
        for i in range(j):
            v -= (q[:, i] @ a[:, j]) * q[:, i]
        q[:, j] = v / np.linalg.norm(v)
    return q


def test_rotation_is_the_positive_diagonal_qr_factor():
    rng = np.random.default_rng(1)
    g = rng.standard_normal((32, 32))
    pi = turbo.rotation(g)
    assert np.abs(pi.T @ pi - np.eye(32)).max() < 1e-12
    r = pi.T @ g
    assert np.abs(np.tril(r, -1)).max() < 1e-10 and np.all(np.diag(r) > 0)
    # Gram-Schmidt on the columns gives the same (unique) factor
    assert np.abs(_gram_schmidt(g) - pi).max() < 1e-9


def test_rotation_preserves_norms_and_spreads_outliers():
    rng = np.random.default_rng(2)
    pi = turbo.rotation(rng.standard_normal((128, 128)))
    x = rng.standard_normal((200, 128))
    x[:, [5, 77]] *= 20.0
    y = x @ pi.T
    assert np.allclose(np.linalg.norm(x, axis=1), np.linalg.norm(y, axis=1))
    ratio = lambda v: np.abs(v).max(axis=1) / np.sqrt((v * v).mean(axis=1))
    assert np.median(ratio(x)) > 7.0 and np.median(ratio(y)) < 4.0


def _fwht(x):
    """Textbook in-place fast Walsh-Hadamard transform (butterflies of span
    1, 2, 4, ...) along the last axis, unnormalised."""
    x = np.array(x, np.float64)
    n = x.shape[-1]
    h = 1
    while h < n:
        for i in range(0, n, 2 * h):
            a = x[..., i:i + h].copy()
            b = x[..., i + h:i + 2 * h].copy()
            x[..., i:i + h] = a + b
            x[..., i + h:i + 2 * h] = a - b
        h *= 2
    return x


@pytest.mark.parametrize("d", [1, 2, 4, 64, 128])
def test_wht_rotation_is_scipys_hadamard_normalised(d):
    from scipy.linalg import hadamard
    assert np.array_equal(turbo.rotation_wht(d) * math.sqrt(d), hadamard(d).astype(np.float64))


def test_wht_rotation_is_an_orthogonal_involution_and_the_fast_transform():
    pi = turbo.rotation_wht(128)
    assert np.abs(pi.T @ pi - np.eye(128)).max() < 1e-14
    assert np.abs(pi @ pi - np.eye(128)).max() < 1e-14          # symmetric: its own inverse
    rng = np.random.default_rng(5)
    x = rng.standard_normal((7, 128))
    assert np.abs(x @ pi.T - _fwht(x) / math.sqrt(128)).max() < 1e-12


def test_wht_rotation_spreads_an_outlier():
    pi = turbo.rotation_wht(128)
    # a single spike becomes a flat vector of the same norm
    y = pi @ np.eye(128)[:, 37]
    assert np.allclose(np.abs(y), 1 / math.sqrt(128))
    rng = np.random.default_rng(6)
    x = rng.standard_normal((200, 128))
    x[:, [5, 77]] *= 20.0
    y = x @ pi.T
    ratio = lambda v: np.abs(v).max(axis=1) / np.sqrt((v * v).mean(axis=1))
    assert np.allclose(np.linalg.norm(x, axis=1), np.linalg.norm(y, axis=1))
    assert np.median(ratio(x)) > 7.0 and np.median(ratio(y)) < 4.0
    with pytest.raises(ValueError):
        turbo.rotation_wht(96)


# ------------------------------------------------------------------ quantizer
def _params(d=128, m=128, seed=3):
    rng = np.random.default_rng(seed)
    pi = turbo.rotation(rng.standard_normal((d, d)))
    s = rng.standard_normal((m, d)).astype(np.float32).astype(np.float64)
    lv, th = turbo.deployed_codebook(d)
    return pi, s, lv, th


def test_zero_vector():
    pi, s, lv, th = _params()
    out = turbo.quantize(np.zeros((1, 128)), pi, lv, th, s)
    assert np.all(out["codes"] == 3) and out["n"][0] == 0 and out["gamma"][0] == 0


def test_scaled_codebook_direction_has_closed_form_codes_gamma_and_signs():
    """x = n Pi^T (c_k / ||c_k||) for a chosen code vector k: the rotated unit
    vector is the codebook point c_k rescaled, so every coordinate stays in its
    own cell (each is chosen at least 1e-3 from both thresholds of its cell),
    the codes come back as k, the residual is e = c_k (1/||c_k|| - 1), gamma =
    n |1 - ||c_k|||, and the sketch signs are those of (S c_k) (1/||c_k|| - 1).
    A transposed Pi, a residual taken in the wrong space, a dropped norm or a
    flipped sign convention each break one of these."""
    pi, s, lv, th = _params()
    rng = np.random.default_rng(4)
    edges = np.concatenate([[-np.inf], th, [np.inf]])
    n = np.array([0.5, 1.0, 3.0, 10.0, 100.0])
    checked = 0
    while checked < len(n):
        k = rng.integers(0, 8, 128)
        ck = lv[k]
        norm = np.linalg.norm(ck)
        y = ck / norm
        # every coordinate at least 1e-3 inside its cell, away from ties
        if np.any(y - edges[k] < 1e-3) or np.any(edges[k + 1] - y < 1e-3):
            continue
        x = n[checked] * (y @ pi)              # Pi^T y as a row vector
        out = turbo.quantize(x[None, :], pi, lv, th, s)
        assert np.array_equal(out["codes"][0], k.astype(np.uint8))
        assert abs(out["n_exact"][0] - n[checked]) <= 1e-12 * n[checked]
        gamma = n[checked] * abs(1.0 - norm)
        assert abs(out["gamma_exact"][0] - gamma) <= 1e-9 * n[checked]
        e_dir = (s @ ck) * (1.0 / norm - 1.0)
        clear = np.abs(e_dir) > 1e-9
        assert np.array_equal(out["signs"][0][clear], (e_dir[clear] >= 0).astype(np.uint8))
        checked += 1


def _turbo_scratch(kb, vb, S0, S, R, G, params):
    """Closed-form state of a row after a prefill of S0 tokens and S - S0
    appends: the window flushes G tokens each time it reaches R + G, so the
    quantized length, window length and ring head follow from the counts, and
    the quantized tokens are the first tq ones, quantized from scratch."""
    pi, s, lv, th = params
    tq0 = G * (max(0, S0 - R) // G)
    r0 = S0 - tq0
    n = S - S0
    flushes = (r0 + n - R) // G if r0 + n >= R + G else 0
    tq = tq0 + G * flushes
    head = (G * flushes) % (R + G)
    k = decode16(kb[:tq], "fp16")
    v = decode16(vb[:tq], "fp16")
    return tq, S - tq, head, turbo.quantize(k, pi, lv, th, s), turbo.quantize(v, pi, lv, th)


@pytest.mark.parametrize("G,R,steps", [(4, 4, 14), (4, 8, 14), (32, 32, 70), (32, 128, 80)])
def test_turbo_row_window_bookkeeping_brute_force(G, R, steps):
    """Every prefill length up to ~R + 2G (and the boundary lengths) followed by
    every append count up to `steps`, on d = m = 8 (the row model does not
    depend on d): T_q, r, the ring head and the window tokens equal the closed
    form, and the quantized tokens equal turbo.quantize applied from scratch to
    the first T_q tokens."""
    d = 8
    rng = np.random.default_rng(7)
    pi = turbo.rotation(rng.standard_normal((d, d)))
    s = rng.standard_normal((d, d))
    lv, th = turbo.deployed_codebook(d)
    params = (pi, s, lv, th)
    lens = sorted(set(list(range(0, R + 2 * G + 2, 1 if G == 4 else 7)) +
                      [R - 1, R, R + 1, R + G - 1, R + G, R + G + 1, 2 * R + G + 5]))
    for S0 in [x for x in lens if x >= 0]:
        total = S0 + steps
        kb = rng.standard_normal((total, d)).astype(np.float16).view(np.uint16)
        vb = rng.standard_normal((total, d)).astype(np.float16).view(np.uint16)
        row = turbo_cache.TurboRow(d, R, "fp16", pi, s, lv, th, G=G)
        row.prefill(kb[:S0], vb[:S0])
        for n in range(0, steps + 1):
            if n:
                row.append(kb[S0 + n - 1], vb[S0 + n - 1])
            S = S0 + n
            tq, r, head, kq, vq = _turbo_scratch(kb, vb, S0, S, R, G, params)
            assert (row.tq, row.r, row.head) == (tq, r, head), (S0, n)
            if S >= R:
                assert R <= row.r < R + G
            idx = (head + np.arange(r)) % (R + G)
            assert np.array_equal(row.ring_k[idx], kb[tq:S]) and np.array_equal(row.ring_v[idx], vb[tq:S])
            wk, wv = row.window_bits()
            assert np.array_equal(wk, kb[tq:S]) and np.array_equal(wv, vb[tq:S])
            for key in ("codes", "n", "gamma", "signs"):
                assert np.array_equal(row.kq[key], kq[key]), (S0, n, key)
            for key in ("codes", "n"):
                assert np.array_equal(row.vq[key], vq[key]), (S0, n, key)


def test_tie_goes_to_lower_index():
    _, _, lv, th = _params()
    assert turbo.codes_of(np.array([th[2]]), th)[0] == 2
    assert turbo.codes_of(np.array([np.nextafter(th[2], 1)]), th)[0] == 3


def test_qjl_estimator_is_unbiased_monte_carlo():
    """Over random Gaussian sketches S (m rows), sqrt(pi/2)/m ||e|| <S q, sign(S e)>
    has mean <q, e> and variance at most pi/(2m) ||q||^2 ||e||^2."""
    rng = np.random.default_rng(5)
    d, m, trials = 32, 16, 20000
    q = rng.standard_normal(d)
    e = rng.standard_normal(d) * 0.3
    est = np.empty(trials)
    for i in range(trials):
        S = rng.standard_normal((m, d))
        est[i] = turbo.qjl_constant(m) * np.linalg.norm(e) * ((S @ q) @ np.sign(S @ e))
    true = q @ e
    se = est.std() / math.sqrt(trials)
    assert abs(est.mean() - true) < 4 * se
    assert est.var() <= math.pi / (2 * m) * (q @ q) * (e @ e) * 1.05


def test_sketch_correction_removes_quantizer_shrinkage():
    """The Lloyd-Max quantizer shrinks inner products: the regression slope of
    <Pi q, c_hat> n on <q, k> is about 1 - MSE(N(0,1)) = 0.9655; adding the QJL
    term makes the estimate unbiased, slope 1."""
    pi, s, lv, th = _params()
    rng = np.random.default_rng(6)
    k = rng.standard_normal((6000, 128))
    q = rng.standard_normal((8, 128))
    kq = turbo.quantize(k, pi, lv, th, s)
    with_qjl = turbo.scores_quantized(q, pi, s, lv, kq, 1.0).ravel()
    no_qjl = (((q @ pi.T) @ (lv[kq["codes"]].T)) * kq["n"][None, :]).ravel()
    exact = (q @ k.T).ravel()
    slope = lambda est: float(est @ exact / (exact @ exact))
    c, t = turbo.lloyd_max_gaussian(8)
    assert abs(slope(no_qjl) - (1 - turbo.gaussian_mse(c, t))) < 0.01
    assert abs(slope(with_qjl) - 1.0) < 0.01


def test_window_only_attention_is_plain_softmax():
    pi, s, lv, th = _params(d=128)
    rng = np.random.default_rng(7)
    kb = rng.standard_normal((20, 128)).astype(np.float16).view(np.uint16)
    vb = rng.standard_normal((20, 128)).astype(np.float16).view(np.uint16)
    row = turbo_cache.TurboRow(128, 128, "fp16", pi, s, lv, th)
    row.prefill(kb, vb)
    q = rng.standard_normal((4, 128)).astype(np.float16)
    got = row.attention(q.view(np.uint16), 0.1)
    K = kb.view(np.float16).astype(np.float64)
    V = vb.view(np.float16).astype(np.float64)
    sc = 0.1 * q.astype(np.float64) @ K.T
    p = np.exp(sc - sc.max(1, keepdims=True))
    assert np.abs(got - (p @ V) / p.sum(1, keepdims=True)).max() < 1e-12


def test_quantized_attention_close_to_exact_attention():
    """3-bit codes + QJL keep the attention output near the unquantized one."""
    pi, s, lv, th = _params()
    rng = np.random.default_rng(8)
    kb = rng.standard_normal((320, 128)).astype(np.float16).view(np.uint16)
    vb = rng.standard_normal((320, 128)).astype(np.float16).view(np.uint16)
    row = turbo_cache.TurboRow(128, 128, "fp16", pi, s, lv, th)
    row.prefill(kb, vb)
    assert row.tq == 192
    q = rng.standard_normal((4, 128)).astype(np.float16)
    got = row.attention(q.view(np.uint16), 1 / math.sqrt(128))
    K = kb.view(np.float16).astype(np.float64)
    V = vb.view(np.float16).astype(np.float64)
    sc = q.astype(np.float64) @ K.T / math.sqrt(128)
    p = np.exp(sc - sc.max(1, keepdims=True))
    exact = (p @ V) / p.sum(1, keepdims=True)
    assert np.linalg.norm(got - exact) / np.linalg.norm(exact) < 0.2


# ------------------------------------------------------------------ layout
def test_layout_round_trip_and_sizes():
    rng = np.random.default_rng(9)
    T = 96
    kc = rng.integers(0, 8, (T, 128)).astype(np.uint8)
    vc = rng.integers(0, 8, (T, 128)).astype(np.uint8)
    ks = rng.integers(0, 2, (T, 128)).astype(np.uint8)
    kn, kg, vn = fp16_round(rng.uniform(0, 50, T)), fp16_round(rng.uniform(0, 5, T)), fp16_round(rng.uniform(0, 50, T))
    rec = turbo_cache.pack_tbs(kc, kn, kg, ks, vc, vn)
    assert rec.shape == (3, 4032)
    for a, b in zip(turbo_cache.unpack_tbs(rec), (kc, kn, kg, ks, vc, vn)):
        assert np.array_equal(a, b)
    # 126 bytes per token and kv head
    assert turbo_cache.TB_BYTES / 32 == 126


def test_layout_hand_worked_positions():
    """Key token 9, coordinate 3: nt 1, gr 1, kt 0, rho 0, tc 1, e 1 -> lane 5,
    slot 16, word 3, field 1 -> bit 6 + 3 = 9, byte 16*5 + 4*3 = 92.
    Value token 9, coordinate 3: kt 0, rho 1, tc 0, e 1; nt 0, gr 3 -> lane 12,
    slot 1, word 0, field 1 -> bit 9, byte 16*12 = 192.
    Sign row 19 of token 9: kt 1, rho 0, tc 1, e 1 -> lane 5, slot 18, word 1,
    bit 2 + 16 = 18, byte 16*5 + 4 = 84."""
    off, bit = turbo_cache.key_code_map()
    assert (off[9, 3], bit[9, 3]) == (92, 9)
    off, bit = turbo_cache.value_code_map()
    assert (off[9, 3], bit[9, 3]) == (192, 9)
    off, bit = turbo_cache.sign_map()
    assert (off[9, 19], bit[9, 19]) == (84, 18)
    # slot 62 of lane 0 (key pair nt 3, kt 7, rho 0) lives in word 12: byte 1536
    off, bit = turbo_cache.key_code_map()
    assert (off[24, 112], bit[24, 112]) == (1536, 12)
