"""The fused decode step (kvq_append_decode) against the two-call step.

A step of kvq_append_decode must leave the cache exactly as kvq_append_token
does and return exactly what kvq_decode_attention returns after it: the same
kernels' arithmetic reads the same values, only the new token comes from the
input instead of the residual window.  Runs cross window flushes (where the
fused call falls back to quantize-then-attend) and window starts; KIVI steps
are also checked against the float64 oracle."""
import numpy as np
import pytest
import torch

from gpu_util import check_row_attention, check_row_bits, gpu_prefill, oracle_row, to_dev
from quantized_kv_cache_18_b200 import workloads as W
from quantized_kv_cache_18_b200.cache import QuantizedKVCache, config_from_workload, turbo_setup_from_workload

pytestmark = pytest.mark.gpu


def _same_state(a, b, unit):
    """Same counters, the same written records (unit = tokens per record) and
    the same valid window slots; unwritten bytes of the buffers are not state."""
    assert (a.seq_len, a.quantized_len, a.window_len, a.window_head) == \
        (b.seq_len, b.quantized_len, b.window_len, b.window_head)
    n = a.quantized_len // unit
    assert torch.equal(a.records_view()[:, :n], b.records_view()[:, :n])
    cap = a.ring_view().shape[2]
    idx = torch.tensor([(a.window_head + i) % cap for i in range(a.window_len)], device=a.buf.device,
                       dtype=torch.long)
    assert torch.equal(a.ring_view()[:, :, idx], b.ring_view()[:, :, idx])


@pytest.mark.parametrize("name,kw,S,steps", [
    ("tiny", dict(), 100, 70),            # R = G = 32: flushes at r = 64
    ("tiny", dict(), 1, 40),              # the window starts with one token
    ("8b2", dict(batch=2), 1000, 40),     # token-major kernel, GQA 4
    ("8b4", dict(batch=2), 700, 70),      # 4-bit G 64: a flush inside the run
    ("70b", dict(), 2000, 30),            # head-major kernel, GQA 8, rows split across CTAs
])
def test_fused_step_matches_two_calls_and_oracle(name, kw, S, steps):
    w = W.with_sizes(W.WORKLOADS[name], **kw)
    K, V = W.prefill(w, seq_len=S)
    fused = gpu_prefill(w, K, V, max_seq=S + steps + 1)
    split = gpu_prefill(w, K, V, max_seq=S + steps + 1)
    rows = [(0, 0), (w.batch - 1, w.num_kv_heads - 1)]
    orows = {bh: oracle_row(w, K[bh[0], bh[1]], V[bh[0], bh[1]]) for bh in rows}
    check = {1, 2, steps // 2, steps}
    for i in range(1, steps + 1):
        kn, vn = W.decode_token(w, i)
        q = W.query(w, i)
        qd = to_dev(q)
        out_f = fused.append_attention(to_dev(kn), to_dev(vn), qd)
        split.append(to_dev(kn), to_dev(vn))
        out_s = split.attention(qd)
        torch.cuda.synchronize()
        assert torch.equal(out_f, out_s), f"step {i}: outputs differ"
        for bh, orow in orows.items():
            orow.append(kn[bh], vn[bh])
        if i in check:
            _same_state(fused, split, w.group)
            out = out_f.cpu().numpy()
            g = w.gqa
            for (b, h), orow in orows.items():
                check_row_bits(fused, b * w.num_kv_heads + h, orow)
                check_row_attention(out[b, h * g:(h + 1) * g], orow, q[b, h * g:(h + 1) * g], w)
    assert fused.status() == 0 and split.status() == 0


def _turbo_cache(w, max_seq):
    cache = QuantizedKVCache(config_from_workload(w, max_seq))
    turbo_setup_from_workload(cache, w)
    return cache


@pytest.mark.parametrize("name,S,steps", [("tq", 480, 72), ("tq", 5, 40), ("tqw", 480, 40)])
def test_fused_step_turbo_matches_two_calls(name, S, steps):
    w = W.with_sizes(W.WORKLOADS[name], batch=1, num_kv_heads=2, num_q_heads=8, seq_len=S, decode_steps=steps)
    K, V = W.prefill(w, seq_len=S)
    fused, split = _turbo_cache(w, S + steps + 1), _turbo_cache(w, S + steps + 1)
    for c in (fused, split):
        c.prefill(to_dev(K), to_dev(V))
    for i in range(1, steps + 1):
        kn, vn = W.decode_token(w, i)
        qd = to_dev(W.query(w, i))
        out_f = fused.append_attention(to_dev(kn), to_dev(vn), qd)
        split.append(to_dev(kn), to_dev(vn))
        out_s = split.attention(qd)
        torch.cuda.synchronize()
        assert torch.equal(out_f, out_s), f"step {i}: outputs differ"
    _same_state(fused, split, 32)
    assert fused.status() == 0


def test_fused_step_errors_leave_state_unchanged():
    from quantized_kv_cache_18_b200._lib import KvqError
    w = W.WORKLOADS["tiny"]
    K, V = W.prefill(w, seq_len=100)
    cache = gpu_prefill(w, K, V, max_seq=101)
    kn, vn = W.decode_token(w, 1)
    q = to_dev(W.query(w, 1))
    cache.append_attention(to_dev(kn), to_dev(vn), q)
    before = (cache.seq_len, cache.quantized_len, cache.window_len, cache.window_head)
    with pytest.raises(KvqError):
        cache.append_attention(to_dev(kn), to_dev(vn), q)       # would exceed max_seq
    assert (cache.seq_len, cache.quantized_len, cache.window_len, cache.window_head) == before
