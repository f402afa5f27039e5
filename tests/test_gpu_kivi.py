"""GPU parity of the KIVI path against the float64 oracle, through the C ABI.

Packed records and window contents must be bit-exact; attention must agree
within max-abs 2e-3 and relative L2 1e-3 with the oracle's attention over the
same dequantized cache.  Cases span several token blocks with ragged tails,
the window edge cases, every supported GQA width, both bit widths, and the
full-size workloads on sampled (batch, kv-head) rows."""
import numpy as np
import pytest
import torch

from gpu_util import check_row_attention, check_row_bits, gpu_prefill, oracle_row, to_dev
from quantized_kv_cache_18_b200 import workloads as W
from quantized_kv_cache_18_b200.cache import QuantizedKVCache, config_from_workload

pytestmark = pytest.mark.gpu


def _run_case(w, S, rows=None, steps=(), check_steps=None):
    K, V = W.prefill(w, seq_len=S)
    cache = gpu_prefill(w, K, V, max_seq=S + max(len(steps), 1) + 1)
    all_rows = [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]
    rows = all_rows if rows is None else rows
    orows = {bh: oracle_row(w, K[bh[0], bh[1]], V[bh[0], bh[1]]) for bh in rows}

    def check(step):
        q = W.query(w, step)
        out = cache.attention(to_dev(q)).cpu().numpy()
        torch.cuda.synchronize()
        for (b, h), orow in orows.items():
            ri = b * w.num_kv_heads + h
            check_row_bits(cache, ri, orow)
            g = w.gqa
            check_row_attention(out[b, h * g:(h + 1) * g], orow, q[b, h * g:(h + 1) * g], w)

    check(0)
    for i, _ in enumerate(steps, start=1):
        kn, vn = W.decode_token(w, i)
        cache.append(to_dev(kn), to_dev(vn))
        for (b, h), orow in orows.items():
            orow.append(kn[b, h], vn[b, h])
        if check_steps is None or i in check_steps:
            check(i)
    assert cache.status() == 0
    return cache


def test_tiny_prefill_and_attention():
    _run_case(W.WORKLOADS["tiny"], 512)


def test_tiny_append_across_flushes():
    # R = G = 32: window 32..63 tokens, a flush every 32 steps
    w = W.WORKLOADS["tiny"]
    _run_case(w, 512, steps=range(100), check_steps={1, 31, 32, 33, 63, 64, 65, 96, 100})


@pytest.mark.parametrize("S", [1, 5, 31, 32, 33, 63, 64, 65, 96, 97])
def test_tiny_window_edges(S):
    _run_case(W.WORKLOADS["tiny"], S, steps=range(40), check_steps={1, 2, 31, 32, 33, 40})


@pytest.mark.parametrize("name,kw,S", [
    ("8b2", dict(batch=2), 1000),                                  # 27 groups + 136 window tokens
    ("8b4", dict(batch=2), 700),                                   # G 64: 8 groups + 188 window tokens
    ("70b", dict(), 4000),                                         # GQA 8
    ("8b2", dict(batch=1, num_q_heads=8), 777),                    # GQA 1
    ("8b2", dict(batch=1, num_q_heads=16), 777),                   # GQA 2
    ("tiny", dict(bits=4), 700),                                   # d 64, 4-bit, G 32
    ("tiny", dict(bits=4, group=64, residual=64), 700),            # d 64, 4-bit, G 64
    ("8b2", dict(batch=1, group=64, residual=128), 901),           # 2-bit, G 64
    ("8b4", dict(batch=1, group=32), 901),                         # 4-bit, G 32
])
def test_shapes(name, kw, S):
    w = W.with_sizes(W.WORKLOADS[name], **kw)
    _run_case(w, S)


@pytest.mark.parametrize("name,kw,S,steps", [
    ("8b4", dict(batch=2), 700, 130),    # flushes at steps where r reaches 192
    ("70b", dict(), 2000, 70),
])
def test_append_shapes(name, kw, S, steps):
    w = W.with_sizes(W.WORKLOADS[name], **kw)
    _run_case(w, S, steps=range(steps), check_steps={1, steps // 2, steps})


def test_fp16_and_bf16_give_same_path_on_same_values():
    """Inputs exactly representable in both formats (small integers / 8) give
    identical records in fp16 and bf16 caches."""
    w16 = W.with_sizes(W.WORKLOADS["tiny"], dtype="fp16")
    wbf = W.with_sizes(W.WORKLOADS["tiny"], dtype="bf16")
    rng = np.random.default_rng(0)
    x = (rng.integers(-64, 64, (1, 2, 300, 64)) / 8.0).astype(np.float32)
    k16, kbf = W.to_bits(x, "fp16"), W.to_bits(x, "bf16")
    v16, vbf = W.to_bits(x[..., ::-1].copy(), "fp16"), W.to_bits(x[..., ::-1].copy(), "bf16")
    c1 = gpu_prefill(w16, k16, v16)
    c2 = gpu_prefill(wbf, kbf, vbf)
    ng = c1.quantized_len // w16.group
    assert ng == 8
    assert torch.equal(c1.records_view()[:, :ng], c2.records_view()[:, :ng])


@pytest.mark.parametrize("dtype,bits", [("fp16", 2), ("fp16", 4), ("bf16", 2)])
def test_code_decisions_on_large_offsets_and_ties(dtype, bits):
    """Groups whose zero-point is large against their scale (the fp32 estimate
    of a code is then least accurate) and inputs sitting exactly on rounding
    boundaries (ties, decided half to even) quantize bit-exactly like the
    oracle."""
    w = W.with_sizes(W.WORKLOADS["tiny"], dtype=dtype, bits=bits)
    rng = np.random.default_rng(7)
    S = 300
    x = np.empty((1, 2, S, 64), np.float32)
    # head 0: offsets of 512 / -300 / 1000 with noise a few ulps wide
    for t0, off in ((0, 512.0), (96, -300.0), (192, 1000.0)):
        x[0, 0, t0:t0 + 108] = off + rng.normal(0.0, 1.5, (min(108, S - t0), 64))
    # head 1: values on the grid z + k s / 2 (every other one a tie), z = 512, s = 1
    levels = (1 << bits) - 1
    x[0, 1] = 512.0 + rng.integers(0, 2 * levels + 1, (S, 64)) / 2.0
    x[0, 1, :, 0] = 512.0          # pins min = 512 and max = 512 + levels in every group
    x[0, 1, :, 1] = 512.0 + levels
    k, v = W.to_bits(x, dtype), W.to_bits(x[..., ::-1].copy(), dtype)
    _run_prefill_bits(w, k, v)


@pytest.mark.parametrize("dtype,bits", [("fp16", 2), ("fp16", 4), ("bf16", 2), ("bf16", 4)])
def test_code_decisions_on_tiny_inputs(dtype, bits):
    """Inputs around 1e-6: fp16 subnormals, and for bf16 zero-points and scales
    that fall into fp16's subnormal range (z then differs from the minimum, so
    codes below z and above the top level are clamped).  Bit-exact like the
    oracle."""
    w = W.with_sizes(W.WORKLOADS["tiny"], dtype=dtype, bits=bits)
    rng = np.random.default_rng(13)
    S = 300
    x = rng.normal(0.0, 1.5e-6, (1, 2, S, 64))
    x[0, 1] += 4e-6
    k, v = W.to_bits(x, dtype), W.to_bits(x[..., ::-1].copy(), dtype)
    _run_prefill_bits(w, k, v)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_code_decisions_d128_g64_4bit(dtype):
    """The 4-bit quantizer instance of 64-token records at d = 128 (eight warps
    a CTA), on the inputs of the two tests above: large zero-points against
    the scale and exact ties (even heads: offsets, odd heads: the half-step
    grid), then inputs around 1e-6.  Bit-exact like the oracle."""
    w = W.with_sizes(W.WORKLOADS["8b4"], batch=1, dtype=dtype)
    assert (w.bits, w.group, w.head_dim) == (4, 64, 128)
    rng = np.random.default_rng(11)
    S, H, levels = 400, w.num_kv_heads, 15
    x = np.empty((1, H, S, 128), np.float32)
    for h in range(H):
        if h % 2 == 0:
            for t0, off in ((0, 512.0), (128, -300.0), (256, 1000.0)):
                x[0, h, t0:t0 + 144] = off + rng.normal(0.0, 1.5, (min(144, S - t0), 128))
        else:
            x[0, h] = 512.0 + rng.integers(0, 2 * levels + 1, (S, 128)) / 2.0
            x[0, h, :, 0] = 512.0
            x[0, h, :, 1] = 512.0 + levels
    _run_prefill_bits(w, W.to_bits(x, dtype), W.to_bits(x[..., ::-1].copy(), dtype))
    y = rng.normal(0.0, 1.5e-6, (1, H, S, 128))
    y[0, 1::2] += 4e-6
    _run_prefill_bits(w, W.to_bits(y, dtype), W.to_bits(y[..., ::-1].copy(), dtype))


def _run_prefill_bits(w, K, V):
    cache = gpu_prefill(w, K, V)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            check_row_bits(cache, b * w.num_kv_heads + h, oracle_row(w, K[b, h], V[b, h]))
    assert cache.status() == 0


@pytest.mark.parametrize("bad", [0x7C00, 0x7E00])   # fp16 +inf, nan
def test_nonfinite_input_sets_status_bit(bad):
    w = W.WORKLOADS["tiny"]
    K, V = W.prefill(w, seq_len=256)
    K[0, 1, 3, 5] = bad             # inside the first quantized group
    V[0, 0, 40, 7] = bad            # inside the second
    cache = gpu_prefill(w, K, V)
    bits = cache.status(clear=True)
    assert bits & 1
    assert cache.status() == 0


def test_output_guard_bands_untouched():
    w = W.WORKLOADS["tiny"]
    K, V = W.prefill(w)
    cache = gpu_prefill(w, K, V)
    q = to_dev(W.query(w))
    n = w.batch * w.num_q_heads * w.head_dim
    buf = torch.full((n + 2048,), 12345.0, device="cuda")
    out = buf[1024:1024 + n].view(w.batch, w.num_q_heads, w.head_dim)
    cache.attention(q, out=out)
    torch.cuda.synchronize()
    assert torch.all(buf[:1024] == 12345.0) and torch.all(buf[1024 + n:] == 12345.0)
    assert torch.isfinite(out).all()


def test_capacity_and_state_errors():
    from quantized_kv_cache_18_b200._lib import KvqError
    w = W.WORKLOADS["tiny"]
    K, V = W.prefill(w, seq_len=100)
    cache = gpu_prefill(w, K, V, max_seq=101)
    kn, vn = W.decode_token(w, 1)
    cache.append(to_dev(kn), to_dev(vn))
    with pytest.raises(KvqError):
        cache.append(to_dev(kn), to_dev(vn))           # would exceed max_seq
    with pytest.raises(KvqError):
        cache.prefill(to_dev(K), to_dev(V))            # not empty
    assert cache.seq_len == 101


# ----------------------------------------------------------------- full-size workloads, sampled rows
@pytest.mark.slow
@pytest.mark.parametrize("name,rows", [
    ("8b2", [(0, 0), (7, 3), (15, 7)]),
    ("70b", [(0, 0), (0, 5)]),
])
def test_full_size_prefill_sampled_rows(name, rows):
    w = W.WORKLOADS[name]
    _run_case(w, w.seq_len, rows=rows)


@pytest.mark.slow
def test_full_size_8b4_256_steps_sampled_rows():
    w = W.WORKLOADS["8b4"]
    _run_case(w, w.seq_len, rows=[(0, 0), (33, 4), (63, 7)], steps=range(w.decode_steps),
              check_steps={1, 63, 64, 65, 128, 192, 256})
