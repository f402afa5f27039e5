"""GPU parity of the mixed-format cache (FP8 anchors and window + TQ3 older
tokens, one merged attention) against the float64 oracle (oracle/mixed_cache.py).

FP8 token rows (anchors and window, codes, scale and padding) must be
bit-exact.  TQ3 blocks, including those flushed from FP8 window rows, follow
the TurboQuant ambiguity rule (tests/test_gpu_turbo.py).  Attention must match
within max-abs 2e-3 and relative L2 1e-3, on the GPU's own cache when no code
was decided differently and always on the oracle's blocks written into the
buffer."""
import numpy as np
import pytest
import torch

from gpu_util import to_dev
from oracle import mixed_cache
from quantized_kv_cache_18_b200 import workloads as W
from test_gpu_turbo import check_attention, check_blocks_values, gpu_cache, oracle_params

pytestmark = pytest.mark.gpu

SMALL = W.with_sizes(W.WORKLOADS["tqm"], batch=1, num_kv_heads=2, num_q_heads=8, anchor_tokens=64)


def run_mixed(w, seq_len, appends=0):
    params = oracle_params(w)
    Pi, S_, lv, th = params
    K, V = W.prefill(w, seq_len=seq_len)
    cache = gpu_cache(w, max_seq=seq_len + appends + 1)
    cache.prefill(to_dev(K), to_dev(V))
    rows = {}
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            r = mixed_cache.MixedRow(w.head_dim, w.residual, w.anchor_tokens, w.dtype, Pi, S_, lv, th, G=w.group)
            r.prefill(K[b, h], V[b, h])
            rows[(b, h)] = r
    for step in range(1, appends + 1):
        kn, vn = W.decode_token(w, step)
        cache.append(to_dev(kn), to_dev(vn))
        for (b, h), r in rows.items():
            r.append(kn[b, h], vn[b, h])
    torch.cuda.synchronize()
    assert cache.status() == 0
    any_row = next(iter(rows.values()))
    assert cache.quantized_len == any_row.tq and cache.window_len == any_row.r
    assert cache.window_head == any_row.head
    rec = cache.records_view()
    ring = cache.fp8_ring_view().cpu().numpy()
    anc = cache.anchor_view().cpu().numpy()
    n_tb = any_row.tq // 32
    flips = 0
    for (b, h), r in rows.items():
        ri = b * w.num_kv_heads + h
        for kvi, kv in enumerate("kv"):
            assert np.array_equal(anc[ri, kvi], r.anchor_rows(kv)), f"row {ri} {kv}: anchor rows differ"
            idx = r.window_idx()
            assert np.array_equal(ring[ri, kvi][idx], r.ring_rows(kv)[idx]), f"row {ri} {kv}: window rows differ"
        if n_tb:
            _, nf = check_blocks_values(rec[ri, :n_tb].cpu().numpy(), w, params, r.k_in, r.v_in)
            flips += nf
    q = W.query(w, 0)
    qd = to_dev(q)
    g = w.gqa
    refs = {(b, h): r.attention(q[b, h * g:(h + 1) * g], w.scale) for (b, h), r in rows.items()}
    if flips == 0:
        out = cache.attention(qd).cpu().numpy()
        for (b, h), ref in refs.items():
            check_attention(out[b, h * g:(h + 1) * g], ref)
    if n_tb:
        for (b, h), r in rows.items():
            rec[b * w.num_kv_heads + h, :n_tb].copy_(torch.from_numpy(r.records()))
    out = cache.attention(qd).cpu().numpy()
    torch.cuda.synchronize()
    assert cache.status() == 0
    return [check_attention(out[b, h * g:(h + 1) * g], ref) for (b, h), ref in refs.items()]


def test_mixed_prefill_only_fp8():
    run_mixed(SMALL, 64 + 100)                    # no TQ3 token: anchors + window only


def test_mixed_prefill_and_appends_across_flushes():
    run_mixed(SMALL, 64 + 500, appends=70)


@pytest.mark.parametrize("seq_len", [64, 65, 64 + 127, 64 + 128, 64 + 161, 64 + 1000])
def test_mixed_window_edges(seq_len):
    run_mixed(SMALL, seq_len, appends=35)


def test_mixed_many_rows_split_across_ctas():
    w = W.with_sizes(W.WORKLOADS["tqm"], batch=4, num_kv_heads=4, num_q_heads=16)
    run_mixed(w, 128 + 3000, appends=3)


def test_mixed_fused_step_is_the_two_calls():
    w = SMALL
    K, V = W.prefill(w, seq_len=64 + 300)
    a, b = gpu_cache(w, max_seq=400), gpu_cache(w, max_seq=400)
    for c in (a, b):
        c.prefill(to_dev(K), to_dev(V))
    for i in range(1, 30):
        kn, vn = W.decode_token(w, i)
        qd = to_dev(W.query(w, i))
        oa = a.append_attention(to_dev(kn), to_dev(vn), qd)
        b.append(to_dev(kn), to_dev(vn))
        ob = b.attention(qd)
        torch.cuda.synchronize()
        assert torch.equal(oa, ob)


def test_mixed_prefill_needs_the_anchors():
    from quantized_kv_cache_18_b200._lib import KvqError
    K, V = W.prefill(SMALL, seq_len=40)
    cache = gpu_cache(SMALL, max_seq=100)
    with pytest.raises(KvqError):
        cache.prefill(to_dev(K), to_dev(V))
