"""Paged caches (a pool of record pages and a per-row block table) against
contiguous caches of the same workload and against the float64 oracle.

Same inputs, same calls: a paged cache must hold bit-identical records (read
through its block table) and window, and return bit-identical attention.  The
block tables are random permutations of the pool, so no row's pages are
adjacent or in order.  After the prefill, at the first step that flushes the
window and at the last step, every row of the paged cache is also checked
against the oracle: records and window bit-exact (TurboQuant blocks under the
ambiguity rule of test_gpu_turbo) and attention within max-abs 2e-3 and rel-L2
1e-3.  A table entry outside the pool must raise KVQ_DEV_BAD_PAGE and be
skipped, never dereferenced."""
import ctypes
import math

import numpy as np
import pytest
import torch

from gpu_util import check_row_attention, oracle_row, to_dev
from quantized_kv_cache_18_b200 import _lib as L
from quantized_kv_cache_18_b200 import workloads as W
from quantized_kv_cache_18_b200.cache import QuantizedKVCache, config_from_workload, turbo_setup_from_workload

pytestmark = pytest.mark.gpu


def _groups_per_row(cfg):
    lay = L.KvqLayout()
    assert L.load().kvq_get_layout(ctypes.byref(cfg), ctypes.byref(lay)) == 0
    return int(lay.groups_per_row)


def _paged(w, max_seq, page_records, seed, spare=3):
    rows = w.batch * w.num_kv_heads
    ppr = math.ceil(_groups_per_row(config_from_workload(w, max_seq)) / page_records)
    num_pages = rows * ppr + spare
    cache = QuantizedKVCache(config_from_workload(w, max_seq, page_records, num_pages))
    assert cache.layout.pages_per_row == ppr
    perm = np.random.default_rng(seed).permutation(num_pages)[:rows * ppr].reshape(rows, ppr)
    cache.set_page_table(torch.tensor(perm, dtype=torch.int32, device="cuda"))
    return cache


def _unit(w):
    return w.group if w.scheme == "kivi" else 32


def _same(paged, flat, w):
    assert (paged.seq_len, paged.quantized_len, paged.window_len, paged.window_head) == \
        (flat.seq_len, flat.quantized_len, flat.window_len, flat.window_head)
    n = flat.quantized_len // _unit(w)
    for r in range(w.batch * w.num_kv_heads):
        assert torch.equal(paged.row_records(r, n), flat.records_view()[r, :n]), f"row {r}: records differ"
    cap = flat.ring_view().shape[2]
    idx = torch.tensor([(flat.window_head + i) % cap for i in range(flat.window_len)], device="cuda",
                       dtype=torch.long)
    assert torch.equal(paged.ring_view()[:, :, idx], flat.ring_view()[:, :, idx])


class _OracleRows:
    """The oracle's rows of a workload, advanced with the same appends, and the
    paged cache's records and window checked against them."""

    def __init__(self, w, K, V):
        self.w = w
        self.rows = [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]
        if w.scheme == "turbo":
            from test_gpu_turbo import oracle_params
            from test_gpu_turbo import oracle_row as tq_row
            self.params = oracle_params(w)
            self.o = {bh: tq_row(w, self.params, K[bh[0], bh[1]], V[bh[0], bh[1]]) for bh in self.rows}
            self.toks = {bh: ([K[bh[0], bh[1]]], [V[bh[0], bh[1]]]) for bh in self.rows}
        else:
            self.o = {bh: oracle_row(w, K[bh[0], bh[1]], V[bh[0], bh[1]]) for bh in self.rows}

    def append(self, kn, vn):
        for (b, h), row in self.o.items():
            row.append(kn[b, h], vn[b, h])
            if self.w.scheme == "turbo":
                self.toks[(b, h)][0].append(kn[b, h][None])
                self.toks[(b, h)][1].append(vn[b, h][None])

    def check_state(self, cache):
        """Records (through the block table) and window of every row; returns
        the number of TurboQuant keys whose codes took the other neighbour."""
        w = self.w
        any_row = next(iter(self.o.values()))
        assert (cache.quantized_len, cache.window_len, cache.window_head) == (any_row.tq, any_row.r, any_row.head)
        n = any_row.tq // _unit(w)
        ring = cache.ring_view().cpu().numpy().view(np.uint16)
        flips = 0
        for (b, h), row in self.o.items():
            ri = b * w.num_kv_heads + h
            if n:
                got = cache.row_records(ri, n).cpu().numpy()
                if w.scheme == "turbo":
                    from test_gpu_turbo import check_blocks
                    kall = np.concatenate(self.toks[(b, h)][0])[:row.tq]
                    vall = np.concatenate(self.toks[(b, h)][1])[:row.tq]
                    flips += check_blocks(got, w, self.params, kall, vall)[1]
                else:
                    assert np.array_equal(got, row.records()), f"row {ri}: records differ from the oracle"
            idx = (row.head + np.arange(row.r)) % row.cap
            assert np.array_equal(ring[ri, 0][idx], row.ring_k[idx]), f"row {ri}: key window differs"
            assert np.array_equal(ring[ri, 1][idx], row.ring_v[idx]), f"row {ri}: value window differs"
        return flips

    def check_attention(self, out, q, flips):
        w, g = self.w, self.w.gqa
        out = out.cpu().numpy()
        for (b, h), row in self.o.items():
            got = out[b, h * g:(h + 1) * g]
            if w.scheme == "turbo":
                if flips == 0:   # same codes on both sides
                    from test_gpu_turbo import check_attention
                    check_attention(got, row.attention(q[b, h * g:(h + 1) * g], w.scale))
            else:
                check_row_attention(got, row, q[b, h * g:(h + 1) * g], w)


@pytest.mark.parametrize("name,kw,S,steps,page_records", [
    ("tiny", dict(), 300, 70, 1),                     # one group per page; flushes
    ("8b2", dict(batch=2), 1500, 40, 4),              # token-major kernel; a stage spans pages
    ("8b4", dict(batch=2), 900, 70, 2),               # 4-bit G 64; a flush
    ("70b", dict(), 3000, 20, 8),                     # head-major kernel, rows split across CTAs
    ("tq", dict(batch=1, num_kv_heads=2, num_q_heads=8), 700, 40, 4),
    ("tqw", dict(batch=1, num_kv_heads=2, num_q_heads=8), 480, 40, 2),
])
def test_paged_cache_matches_contiguous(name, kw, S, steps, page_records):
    w = W.with_sizes(W.WORKLOADS[name], **kw)
    K, V = W.prefill(w, seq_len=S)
    max_seq = S + steps + 1
    flat = QuantizedKVCache(config_from_workload(w, max_seq))
    paged = _paged(w, max_seq, page_records, seed=11)
    for c in (flat, paged):
        if w.scheme == "turbo":
            turbo_setup_from_workload(c, w)
        c.prefill(to_dev(K), to_dev(V))
    _same(paged, flat, w)
    orc = _OracleRows(w, K, V)
    flips = orc.check_state(paged)
    q0 = W.query(w, 0)
    orc.check_attention(paged.attention(to_dev(q0)), q0, flips)
    first_flush = None
    for i in range(1, steps + 1):
        kn, vn = W.decode_token(w, i)
        q = W.query(w, i)
        qd = to_dev(q)
        kd, vd = to_dev(kn), to_dev(vn)
        tq_before = paged.quantized_len
        out_p = paged.append_attention(kd, vd, qd)
        out_f = flat.append_attention(kd, vd, qd)
        orc.append(kn, vn)
        torch.cuda.synchronize()
        assert torch.equal(out_p, out_f), f"step {i}: outputs differ"
        flushed = paged.quantized_len != tq_before
        if (flushed and first_flush is None) or i == steps:
            first_flush = first_flush or (i if flushed else None)
            orc.check_attention(out_p, q, orc.check_state(paged))
    assert first_flush is not None, "the case must cross a flush"
    _same(paged, flat, w)
    assert paged.status() == 0 and flat.status() == 0


def test_bad_page_entry_is_reported_not_dereferenced():
    w = W.with_sizes(W.WORKLOADS["8b2"], batch=1, num_kv_heads=2, num_q_heads=8)
    K, V = W.prefill(w, seq_len=1200)
    cache = _paged(w, 1300, 4, seed=3)
    table = cache.page_table.clone()
    table[1, 2] = cache.cfg.num_pages + 5            # row 1, records 8..11: outside the pool
    cache.set_page_table(table)
    cache.prefill(to_dev(K), to_dev(V))
    bits = cache.status(clear=True)
    assert bits & L.KVQ_DEV_BAD_PAGE
    cache.attention(to_dev(W.query(w, 0)))
    bits = cache.status(clear=True)
    assert bits & L.KVQ_DEV_BAD_PAGE
    # a good table again: the cache works (prefill of a fresh one)
    good = _paged(w, 1300, 4, seed=3)
    good.prefill(to_dev(K), to_dev(V))
    good.attention(to_dev(W.query(w, 0)))
    assert good.status() == 0


def test_paged_calls_need_a_table():
    from quantized_kv_cache_18_b200._lib import KvqError
    w = W.WORKLOADS["tiny"]
    cfg = config_from_workload(w, 600, 2, 40)
    cache = QuantizedKVCache(cfg)
    K, V = W.prefill(w, seq_len=300)
    with pytest.raises(KvqError):
        cache.prefill(to_dev(K), to_dev(V))
