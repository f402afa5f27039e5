"""kvq_decode_attention_static: decode attention for callers that cannot
allocate device memory.

A plugin hosted by a serving engine that owns every device allocation, or a
serving loop that forbids allocator calls once it runs, cannot hand
kvq_decode_attention the scratch workspace it takes.  This entry point uses a
fixed scratch array inside the library instead.  These tests call it through
the C ABI and check it against kvq_decode_attention on two calls in a row;
they pass run alone in a fresh process or after the rest of the suite (the
file sorts last so a stop-at-first-failure run has done everything else)."""
import ctypes

import numpy as np
import pytest
import torch

from gpu_util import ATOL, REL_L2, gpu_prefill, to_dev
from quantized_kv_cache_18_b200 import _lib as L
from quantized_kv_cache_18_b200 import workloads as W
from quantized_kv_cache_18_b200.cache import QuantizedKVCache, make_config, workspace_bytes

pytestmark = pytest.mark.gpu


def _static_call(cache, q, out):
    lib = L.load()
    st = torch.cuda.current_stream()
    return lib.kvq_decode_attention_static(cache.handle, ctypes.c_void_p(q.data_ptr()),
                                           ctypes.c_void_p(out.data_ptr()), ctypes.c_float(cache_scale(cache)),
                                           ctypes.c_void_p(st.cuda_stream))


def cache_scale(cache):
    return 1.0 / np.sqrt(cache.cfg.head_dim)


def _agree(a, b):
    a, b = a.double(), b.double()
    err = (a - b).abs().max().item()
    rel = ((a - b).norm() / b.norm()).item()
    assert err <= ATOL and rel <= REL_L2, (err, rel)


@pytest.mark.parametrize("name,kw,S", [
    ("tiny", dict(), 512),
    ("8b2", dict(batch=2), 1000),
    ("70b", dict(), 5000),
    ("8b4", dict(batch=2), 700),
])
def test_static_entry_point_matches_workspace_entry_point(name, kw, S):
    w = W.with_sizes(W.WORKLOADS[name], **kw)
    K, V = W.prefill(w, seq_len=S)
    cache = gpu_prefill(w, K, V)
    assert workspace_bytes(cache.cfg) <= 4 * 1024 * 1024
    q = to_dev(W.query(w, 3))
    ref = cache.attention(q)
    for _ in range(2):           # two calls in a row share the one scratch array
        out = torch.full_like(ref, float("nan"))
        assert _static_call(cache, q, out) == L.KVQ_OK
        torch.cuda.synchronize()
        _agree(out, ref)
    assert cache.status() == 0


def test_static_entry_point_on_a_turboquant_cache():
    """The TurboQuant workspace is the rotated-query prefix followed by the
    partial slots; the static array holds both.  Two calls in a row against
    kvq_decode_attention and against the float64 oracle over the same codes."""
    from test_gpu_turbo import SMALL, check_attention, gpu_cache, oracle_params
    from test_gpu_turbo import oracle_row as tq_row
    w = W.with_sizes(SMALL, batch=3, num_kv_heads=2, num_q_heads=8, seq_len=1500)
    params = oracle_params(w)
    K, V = W.prefill(w, seq_len=1500)
    cache = gpu_cache(w)
    cache.prefill(to_dev(K), to_dev(V))
    assert workspace_bytes(cache.cfg) <= 4 * 1024 * 1024
    rows = {(b, h): tq_row(w, params, K[b, h], V[b, h]) for b in range(w.batch) for h in range(w.num_kv_heads)}
    n_tb = cache.quantized_len // 32
    rec = cache.records_view()
    for (b, h), row in rows.items():   # the oracle's blocks, so both sides read the same codes
        rec[b * w.num_kv_heads + h, :n_tb].copy_(torch.from_numpy(row.records()))
    qh = W.query(w, 2)
    q = to_dev(qh)
    ref = cache.attention(q)
    g = w.gqa
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        assert _static_call(cache, q, out) == L.KVQ_OK
        torch.cuda.synchronize()
        _agree(out, ref)
        o = out.cpu().numpy()
        for (b, h), row in rows.items():
            check_attention(o[b, h * g:(h + 1) * g], row.attention(qh[b, h * g:(h + 1) * g], w.scale))
    assert cache.status() == 0


def test_static_entry_point_rejects_configs_over_the_limit():
    # (rows + SMs) * g * (d + 4) * 4 bytes of scratch > 4 MiB for 2048 rows of GQA 4, d 128
    cfg = make_config("kivi", 2, 32, 32, 128, 8, 32, 256, 64, "bf16")
    assert workspace_bytes(cfg) > 4 * 1024 * 1024
    cache = QuantizedKVCache(cfg)
    q = torch.zeros((256, 32, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((256, 32, 128), dtype=torch.float32, device="cuda")
    assert _static_call(cache, q, out) == L.KVQ_ERR_CAPACITY


def test_static_entry_point_rejects_null_cache():
    lib = L.load()
    assert lib.kvq_decode_attention_static(None, None, None, ctypes.c_float(1.0), None) == L.KVQ_ERR_INVALID_ARG
