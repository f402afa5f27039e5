"""The bounded waits of the decode kernels and of the tensor-core TurboQuant
quantizer, exercised without a GPU fault.

Every pipeline wait inside a decode launch gives up after a bound; the
launch then sets KVQ_DEV_WAIT_TIMEOUT and finishes without the outputs it
cannot trust, and the GPU context stays usable.  kvq_debug_set_wait_test
shortens the bound and makes CTA 0 withhold the copy of its first stage: a
wait that nothing completes.  These tests check that the status bit is set,
that kvq_get_status(clear) resets the status word and the rows' arrival
counters, and that the next launch matches the float64 oracle again."""
import numpy as np
import pytest
import torch

from gpu_util import check_row_attention, gpu_prefill, oracle_row, to_dev
from quantized_kv_cache_18_b200 import _lib as L
from quantized_kv_cache_18_b200 import workloads as W

pytestmark = pytest.mark.gpu

SHORT_WAIT = 400_000   # SM cycles, about 0.2 ms at the B200's clock


def _timed_out_then_recovers(cache, run_attention, check_output):
    lib = L.load()
    torch.cuda.synchronize()
    assert cache.status() == 0
    L.check(lib.kvq_debug_set_wait_test(SHORT_WAIT, 1), "kvq_debug_set_wait_test")
    try:
        run_attention()
        torch.cuda.synchronize()
    finally:
        L.check(lib.kvq_debug_set_wait_test(0, 0), "kvq_debug_set_wait_test")
    assert cache.status(clear=True) & L.KVQ_DEV_WAIT_TIMEOUT
    assert cache.status() == 0
    for _ in range(2):   # two clean launches: the arrival counters are back at zero
        check_output(run_attention())
        torch.cuda.synchronize()
        assert cache.status() == 0


@pytest.mark.parametrize("name,kw,S", [
    ("70b", dict(), 5000),          # GQA 8: rows split over many CTAs, head-major
    ("8b2", dict(batch=2), 3000),   # GQA 4: token-major
    ("tiny", dict(), 512),          # one CTA per row chunk, fp16
])
def test_kivi_wait_timeout_sets_status_and_recovers(name, kw, S):
    w = W.with_sizes(W.WORKLOADS[name], **kw)
    K, V = W.prefill(w, seq_len=S)
    cache = gpu_prefill(w, K, V)
    q = W.query(w, 2)
    qd = to_dev(q)
    rows = [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]
    orows = {bh: oracle_row(w, K[bh[0], bh[1]], V[bh[0], bh[1]]) for bh in rows}

    def check(out):
        out = out.cpu().numpy()
        g = w.gqa
        for (b, h), orow in orows.items():
            check_row_attention(out[b, h * g:(h + 1) * g], orow, q[b, h * g:(h + 1) * g], w)

    _timed_out_then_recovers(cache, lambda: cache.attention(qd), check)


def test_turbo_wait_timeout_sets_status_and_recovers():
    from test_gpu_turbo import SMALL, check_attention, gpu_cache, oracle_params
    from test_gpu_turbo import oracle_row as tq_row
    w = W.with_sizes(SMALL, batch=2, seq_len=3000)
    params = oracle_params(w)
    K, V = W.prefill(w, seq_len=3000)
    cache = gpu_cache(w)
    cache.prefill(to_dev(K), to_dev(V))
    rows = {(b, h): tq_row(w, params, K[b, h], V[b, h]) for b in range(w.batch) for h in range(w.num_kv_heads)}
    n_tb = cache.quantized_len // 32
    rec = cache.records_view()
    for (b, h), row in rows.items():   # the oracle's blocks: both sides read the same codes
        rec[b * w.num_kv_heads + h, :n_tb].copy_(torch.from_numpy(row.records()))
    q = W.query(w, 1)
    qd = to_dev(q)
    g = w.gqa

    def check(out):
        out = out.cpu().numpy()
        for (b, h), row in rows.items():
            check_attention(out[b, h * g:(h + 1) * g], row.attention(q[b, h * g:(h + 1) * g], w.scale))

    _timed_out_then_recovers(cache, lambda: cache.attention(qd), check)


def test_turbo_quantizer_wait_timeout_sets_status_and_recovers():
    """The tensor-core TurboQuant quantizer: CTA 0 withholds its operand-image
    copy, its mma thread's wait runs out, the CTA stops at a tile boundary and
    sets the status bit; the other CTAs finish.  After a clear, a fresh prefill
    quantizes every block like the oracle."""
    from test_gpu_turbo import SMALL, check_blocks, gpu_cache, oracle_params
    lib = L.load()
    w = W.with_sizes(SMALL, batch=2, seq_len=3000)
    K, V = W.prefill(w, seq_len=3000)
    cache = gpu_cache(w)
    torch.cuda.synchronize()
    assert cache.status() == 0
    L.check(lib.kvq_debug_set_wait_test(SHORT_WAIT, 1), "kvq_debug_set_wait_test")
    try:
        cache.prefill(to_dev(K), to_dev(V))
        torch.cuda.synchronize()
    finally:
        L.check(lib.kvq_debug_set_wait_test(0, 0), "kvq_debug_set_wait_test")
    assert cache.status(clear=True) & L.KVQ_DEV_WAIT_TIMEOUT
    assert cache.status() == 0
    params = oracle_params(w)
    fresh = gpu_cache(w)
    fresh.prefill(to_dev(K), to_dev(V))
    torch.cuda.synchronize()
    assert fresh.status() == 0
    n_tb = fresh.quantized_len // 32
    assert n_tb > 0
    rec = fresh.records_view()
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            check_blocks(rec[b * w.num_kv_heads + h, :n_tb].cpu().numpy(), w, params,
                         K[b, h][:32 * n_tb], V[b, h][:32 * n_tb])


def test_wait_bound_above_default_is_rejected():
    lib = L.load()
    assert lib.kvq_debug_set_wait_test(1 << 40, 0) == L.KVQ_ERR_INVALID_ARG
    assert lib.kvq_debug_set_wait_test(0, 0) == L.KVQ_OK
