"""GPU parity of the TurboQuant-style path (kvq_turbo_setup, prefill/append
quantization, decode attention) against the float64 oracle.

Codes, sketch signs, norms and gamma are decided on the GPU from fp32 (codes,
signs) or fp64 (norms) arithmetic and in float64 by the oracle.  They must be
equal except where the oracle's exact value lies within a bound of a decision
boundary that covers the GPU's rounding error:
  * code of y_c: |y_c - threshold| < EPS_Y, with EPS_Y >= the fp32 error of a
    128-term dot product of unit vectors, ~130 * 2^-24 = 7.7e-6; either
    neighbouring code is then accepted;
  * a token with a code that took the other neighbour has a different
    residual e, so its gamma and signs are not compared (only counted);
  * sign bit: |(S e)_i| < EPS_SE;
  * fp16 n: both sides compute the norm in fp64 from the 16-bit inputs
    (relative error below 128 * 2^-53, about 1.4e-14), so n must be
    bit-exact unless the exact norm lies within EPS_N = 1e-12 (relative) of
    an fp16 rounding midpoint;
  * fp16 gamma = n ||y - c_hat||: the GPU's y has an error below EPS_Y per
    coordinate, so ||e|| is off by at most sqrt(d) EPS_Y (triangle
    inequality); a gamma may differ from the oracle's only as the other fp16
    neighbour of the exact value, when the exact value lies within
    n sqrt(d) EPS_Y of the midpoint between the two.
Every code and sign inside its window, and every norm or gamma that actually
differs, counts as ambiguous; the ambiguous fraction of all these decisions
must stay under 0.5 %.  Attention is
compared on a cache whose packed blocks are the oracle's own (written into the
buffer), so both sides read the same codes, within max-abs 2e-3 and rel-L2
1e-3; with no code decided differently the GPU's own cache is compared too.
"""
import math

import numpy as np
import pytest
import torch

from oracle import turbo, turbo_cache
from oracle.numerics import decode16, fp16_bits
from quantized_kv_cache_18_b200 import workloads as W
from quantized_kv_cache_18_b200._lib import KVQ_DEV_NONFINITE_INPUT
from quantized_kv_cache_18_b200.cache import QuantizedKVCache, config_from_workload, turbo_setup_from_workload

from gpu_util import ATOL, REL_L2, to_dev

pytestmark = pytest.mark.gpu

EPS_Y = 1e-5
EPS_SE = 1e-4
EPS_N = 1e-12

TQ = W.WORKLOADS["tq"]
SMALL = W.with_sizes(TQ, batch=1, num_kv_heads=2, num_q_heads=8, seq_len=480, decode_steps=72)


# ------------------------------------------------------------------ helpers
def oracle_params(w):
    Pi = (turbo.rotation_wht(w.head_dim) if w.rotation == "wht"
          else turbo.rotation(W.gaussian_matrix(w, "rot", w.head_dim, w.head_dim)))
    S = W.gaussian_matrix(w, "qjl", w.qjl_dim, w.head_dim).astype(np.float64)
    lv, th = turbo.deployed_codebook(w.head_dim)
    return Pi, S, lv, th


def gpu_cache(w, max_seq=None):
    cache = QuantizedKVCache(config_from_workload(w, max_seq))
    turbo_setup_from_workload(cache, w)
    return cache


def oracle_row(w, params, kb, vb):
    Pi, S, lv, th = params
    row = turbo_cache.TurboRow(w.head_dim, w.residual, w.dtype, Pi, S, lv, th, G=w.group)
    row.prefill(kb, vb)
    return row


def _near_fp16_midpoint(x, tol):
    """True where float64 x lies within `tol` (absolute, scalar or per value)
    of a midpoint between two adjacent fp16 values."""
    x = np.abs(np.asarray(x, np.float64))
    h = x.astype(np.float16).astype(np.float64)
    nxt = np.nextafter(h.astype(np.float16), np.float16(np.inf)).astype(np.float64)
    prv = np.nextafter(h.astype(np.float16), np.float16(0)).astype(np.float64)
    mids = np.stack([0.5 * (h + nxt), 0.5 * (h + prv)])
    return np.any(np.abs(mids - x) <= tol, axis=0)


def _fp16_neighbours(a, b):
    """True where fp16 values a and b (float64 arrays) are equal or adjacent."""
    ua = np.abs(fp16_bits(a).astype(np.int64))
    ub = np.abs(fp16_bits(b).astype(np.int64))
    return np.abs(ua - ub) <= 1


def check_blocks(got_rec, w, params, k_bits, v_bits):
    """got_rec: uint8 [n_tb][4032] from the GPU; k_bits, v_bits: the quantized
    tokens (uint16 [32 n_tb][d]).  Returns the ambiguous fraction."""
    return check_blocks_values(got_rec, w, params, decode16(k_bits, w.dtype), decode16(v_bits, w.dtype))


def check_blocks_values(got_rec, w, params, k, v):
    """As check_blocks, with the quantized tokens as float64 vectors [32 n_tb][d]."""
    Pi, S, lv, th = params
    kq = turbo.quantize(k, Pi, lv, th, S)
    vq = turbo.quantize(v, Pi, lv, th)
    kc, kn, kg, ks, vc, vn = turbo_cache.unpack_tbs(got_rec, w.head_dim, w.qjl_dim)
    n_amb = 0
    n_dec = 0
    flipped_tok = np.zeros(kc.shape[0], bool)
    for codes, q in ((kc, kq), (vc, vq)):
        dist = np.min(np.abs(q["y"][..., None] - th), axis=-1)
        amb = dist < EPS_Y
        diff = codes != q["codes"]
        assert not np.any(diff & ~amb), f"{int(np.sum(diff & ~amb))} codes differ away from a threshold"
        assert np.all(np.abs(codes[diff].astype(int) - q["codes"][diff].astype(int)) == 1)
        n_amb += int(amb.sum())
        n_dec += amb.size
        if q is kq:
            flipped_tok = diff.any(axis=1)
    # norms: fp16 of an fp64 norm on both sides
    for got, q in ((kn, kq), (vn, vq)):
        bad = fp16_bits(got) != fp16_bits(q["n"])
        assert not np.any(bad & ~_near_fp16_midpoint(q["n_exact"], EPS_N * q["n_exact"])), "norm differs"
        n_amb += int(bad.sum())
        n_dec += bad.size
    # gamma and signs of the tokens whose key codes all agree
    ok = ~flipped_tok
    badg = (fp16_bits(kg) != fp16_bits(kq["gamma"])) & ok
    g_tol = kq["n_exact"] * math.sqrt(w.head_dim) * EPS_Y
    assert not np.any(badg & ~(_near_fp16_midpoint(kq["gamma_exact"], g_tol) &
                               _fp16_neighbours(kg, kq["gamma"]))), "gamma differs"
    n_amb += int(badg.sum())
    n_dec += int(ok.sum())
    amb_s = np.abs(kq["se"]) < EPS_SE
    bads = (ks != kq["signs"]) & ok[:, None]
    assert not np.any(bads & ~amb_s), f"{int(np.sum(bads & ~amb_s))} sign bits differ away from 0"
    n_amb += int(amb_s.sum())
    n_dec += amb_s.size
    frac = n_amb / n_dec
    assert frac < 5e-3, f"ambiguous fraction {frac:.2e}"
    return frac, int(flipped_tok.sum())


def check_attention(out, ref):
    err = np.abs(out.astype(np.float64) - ref)
    rel = np.linalg.norm(out.astype(np.float64) - ref) / np.linalg.norm(ref)
    assert err.max() <= ATOL, f"max-abs {err.max():.3e} > {ATOL}"
    assert rel <= REL_L2, f"rel-L2 {rel:.3e} > {REL_L2}"
    return float(err.max()), float(rel)


def run_case(w, seq_len, appends=0, check_e2e=True):
    """Prefill seq_len tokens, then `appends` decode tokens; check blocks, window
    and attention of every row."""
    params = oracle_params(w)
    K, V = W.prefill(w, seq_len=seq_len)
    cache = gpu_cache(w, max_seq=seq_len + appends + 1)
    cache.prefill(to_dev(K), to_dev(V))
    rows = {}
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            rows[(b, h)] = oracle_row(w, params, K[b, h], V[b, h])
    allk = {key: [K[key[0], key[1]]] for key in rows}
    allv = {key: [V[key[0], key[1]]] for key in rows}
    for step in range(1, appends + 1):
        kn, vn = W.decode_token(w, step)
        cache.append(to_dev(kn), to_dev(vn))
        for (b, h), row in rows.items():
            row.append(kn[b, h], vn[b, h])
            allk[(b, h)].append(kn[b, h][None])
            allv[(b, h)].append(vn[b, h][None])
    torch.cuda.synchronize()
    assert cache.status() == 0
    flips = 0
    any_row = next(iter(rows.values()))
    assert cache.quantized_len == any_row.tq and cache.window_len == any_row.r
    assert cache.window_head == any_row.head
    rec = cache.records_view()
    ring = cache.ring_view().cpu().numpy().view(np.uint16)
    n_tb = any_row.tq // 32
    for (b, h), row in rows.items():
        ri = b * w.num_kv_heads + h
        if n_tb:
            kall = np.concatenate(allk[(b, h)])[:row.tq]
            vall = np.concatenate(allv[(b, h)])[:row.tq]
            _, nf = check_blocks(rec[ri, :n_tb].cpu().numpy(), w, params, kall, vall)
            flips += nf
        idx = (row.head + np.arange(row.r)) % row.cap
        assert np.array_equal(ring[ri, 0][idx], row.ring_k[idx])
        assert np.array_equal(ring[ri, 1][idx], row.ring_v[idx])
    q = W.query(w, 0)
    qd = to_dev(q)
    refs = {}
    for (b, h), row in rows.items():
        g = w.gqa
        refs[(b, h)] = row.attention(q[b, h * g:(h + 1) * g], w.scale)
    if check_e2e and flips == 0:
        out = cache.attention(qd).cpu().numpy()
        for (b, h), ref in refs.items():
            check_attention(out[b, h * w.gqa:(h + 1) * w.gqa], ref)
    # the oracle's own blocks in the buffer: the same codes on both sides
    if n_tb:
        for (b, h), row in rows.items():
            rec[b * w.num_kv_heads + h, :n_tb].copy_(torch.from_numpy(row.records()))
    out = cache.attention(qd).cpu().numpy()
    torch.cuda.synchronize()
    assert cache.status() == 0
    res = []
    for (b, h), ref in refs.items():
        res.append(check_attention(out[b, h * w.gqa:(h + 1) * w.gqa], ref))
    return res


# ------------------------------------------------------------------ setup
def test_setup_tables_match_the_oracle():
    w = SMALL
    cache = gpu_cache(w)
    torch.cuda.synchronize()
    assert cache.status() == 0
    p = cache.params_view().cpu().numpy()
    Pi, S, lv, th = oracle_params(w)
    d = w.head_dim
    f32 = p[:3 * d * d * 4].view(np.float32)
    gpi, gpit, gst = f32[:d * d].reshape(d, d), f32[d * d:2 * d * d].reshape(d, d), f32[2 * d * d:].reshape(d, d)
    # Householder QR in fp64, then fp32: within a couple of fp32 ulps of the oracle's factor
    assert np.abs(gpi.astype(np.float64) - Pi).max() < 1e-6
    assert np.array_equal(gpit, gpi.T)
    assert np.array_equal(gst, W.gaussian_matrix(w, "qjl", w.qjl_dim, d).T)
    off = 3 * d * d * 4
    levels = p[off:off + 32].view(np.float32)
    thr = p[off + 32:off + 64].view(np.float32)
    lv16 = p[off + 64:off + 80].view(np.uint16)
    lut = p[off + 128:off + 384].view(np.uint32)
    assert np.array_equal(levels.astype(np.float64), lv)
    assert np.array_equal(thr[:7].astype(np.float64), th) and np.isinf(thr[7])
    assert np.array_equal(lv16, fp16_bits(lv))
    idx = np.arange(64)
    want = fp16_bits(lv)[idx & 7].astype(np.uint32) | (fp16_bits(lv)[idx >> 3].astype(np.uint32) << 16)
    assert np.array_equal(lut, want)
    # (S Pi)^T: fp64 sums of the fp32 tables, then fp32 -- within a few fp32 ulps of the oracle's S Pi
    spit = p[off + 384:off + 384 + d * d * 4].view(np.float32).reshape(d, d)
    assert np.abs(spit.T.astype(np.float64) - S @ Pi).max() < 2e-5
    # tensor-core operand images: 16 Pi and S split hi + lo, fp16 set then bf16 set, in the
    # no-swizzle K-major layout (core matrix (n/8, k/8) at 2048 (k/8) + 128 (n/8), row n%8 at 16 B)
    img0 = off + 384 + d * d * 4
    n_i, k_i = np.meshgrid(np.arange(d), np.arange(d), indexing="ij")
    pos = ((k_i >> 3) * 2048 + (n_i >> 3) * 128 + (n_i & 7) * 16 + (k_i & 7) * 2) // 2
    for kind, (rn, widen) in enumerate(((_rn_fp16_bits, _fp16_bits_value), (_rn_bf16_bits, _bf16_bits_value))):
        imgs = p[img0 + kind * 4 * 32768: img0 + (kind + 1) * 4 * 32768].view(np.uint16).reshape(4, d * d)
        for j, mat in enumerate((16.0 * gpi, gst.T)):   # B[n][k] = 16 Pi[n][k], S[n][k]
            mat = mat.astype(np.float32)
            hi = rn(mat)
            lo = rn((mat - widen(hi)).astype(np.float32))
            assert np.array_equal(imgs[2 * j][pos], hi), (kind, j, "hi")
            assert np.array_equal(imgs[2 * j + 1][pos], lo), (kind, j, "lo")


def _rn_fp16_bits(x32):
    return x32.astype(np.float16).view(np.uint16)


def _fp16_bits_value(b):
    return b.view(np.float16).astype(np.float32)


def _rn_bf16_bits(x32):
    # round to nearest even on the upper 16 bits of the fp32 pattern (finite inputs)
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _bf16_bits_value(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------------ Walsh-Hadamard rotation
SMALL_WHT = W.with_sizes(SMALL, rotation="wht")


def test_wht_setup_tables_are_exact():
    w = SMALL_WHT
    cache = gpu_cache(w)
    torch.cuda.synchronize()
    assert cache.status() == 0
    p = cache.params_view().cpu().numpy()
    d = w.head_dim
    f32 = p[:3 * d * d * 4].view(np.float32)
    gpi, gpit = f32[:d * d].reshape(d, d), f32[d * d:2 * d * d].reshape(d, d)
    # exactly the oracle's H / sqrt(d) rounded to fp32 (entries +-fp32(1/sqrt(d)))
    assert np.array_equal(gpi, turbo.rotation_wht(d).astype(np.float32))
    assert np.array_equal(gpit, gpi)
    assert np.array_equal(f32[2 * d * d:].reshape(d, d), W.gaussian_matrix(w, "qjl", w.qjl_dim, d).T)


def test_wht_small_prefill_and_appends():
    run_case(SMALL_WHT, 480, appends=72)


@pytest.mark.parametrize("seq_len", [1, 33, 161])
def test_wht_window_edges(seq_len):
    run_case(SMALL_WHT, seq_len, appends=40)


def test_turbo_calls_need_setup():
    from quantized_kv_cache_18_b200._lib import KvqError
    w = SMALL
    cache = QuantizedKVCache(config_from_workload(w))
    K, V = W.prefill(w, seq_len=64)
    with pytest.raises(KvqError):
        cache.prefill(to_dev(K), to_dev(V))


# ------------------------------------------------------------------ quantization + attention
def test_small_prefill():
    run_case(SMALL, 480)


def test_small_appends_cross_flushes():
    # 480 -> T_q = 352, r = 128; 72 appends flush at r = 160 twice
    run_case(SMALL, 480, appends=72)


@pytest.mark.parametrize("seq_len", [1, 31, 32, 127, 128, 129, 159, 160, 161, 192, 200, 4000])
def test_window_edges(seq_len):
    run_case(SMALL, seq_len)


@pytest.mark.parametrize("hq", [2, 4, 8, 16])
def test_gqa_shapes(hq):
    w = W.with_sizes(SMALL, num_kv_heads=2, num_q_heads=hq, batch=3, seq_len=700)
    run_case(w, 700)


def test_fp16_inputs_and_short_window():
    w = W.with_sizes(SMALL, dtype="fp16", residual=32, seq_len=300)
    run_case(w, 300, appends=40)


def test_many_rows_split_across_ctas():
    # more rows than SMs: each CTA spans row boundaries and both parts of rows
    w = W.with_sizes(TQ, batch=20, num_kv_heads=8, num_q_heads=32, seq_len=1000)
    run_case(w, 1000, check_e2e=False)


def test_nonfinite_input_sets_status():
    w = SMALL
    K, V = W.prefill(w, seq_len=64 + w.residual)
    K[0, 1, 5, 7] = 0x7C00 if w.dtype == "fp16" else 0x7F80
    cache = gpu_cache(w)
    cache.prefill(to_dev(K), to_dev(V))
    torch.cuda.synchronize()
    assert cache.status(clear=True) & KVQ_DEV_NONFINITE_INPUT
    assert cache.status() == 0


@pytest.mark.slow
def test_full_tq_sampled_rows():
    """The full 8 x 8 x 32768 workload in the bench's launch configuration;
    blocks and attention of sampled rows."""
    w = TQ
    params = oracle_params(w)
    K, V = W.prefill(w)
    cache = gpu_cache(w)
    cache.prefill(to_dev(K), to_dev(V))
    torch.cuda.synchronize()
    assert cache.status() == 0
    rec = cache.records_view()
    n_tb = cache.quantized_len // 32
    sample = [(0, 0), (3, 5), (7, 7)]
    rows = {}
    for (b, h) in sample:
        row = oracle_row(w, params, K[b, h], V[b, h])
        rows[(b, h)] = row
        ri = b * w.num_kv_heads + h
        check_blocks(rec[ri, :n_tb].cpu().numpy(), w, params, K[b, h][:row.tq], V[b, h][:row.tq])
        rec[ri, :n_tb].copy_(torch.from_numpy(row.records()))
    q = W.query(w, 0)
    out = cache.attention(to_dev(q)).cpu().numpy()
    for (b, h), row in rows.items():
        g = w.gqa
        check_attention(out[b, h * g:(h + 1) * g], row.attention(q[b, h * g:(h + 1) * g], w.scale))
