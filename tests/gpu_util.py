"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare it with the float64 oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import attention as oatt
from oracle.cache import KiviRow
from oracle.numerics import decode16
from quantized_kv_cache_18_b200 import workloads as W
from quantized_kv_cache_18_b200.cache import QuantizedKVCache, config_from_workload

# Attention tolerance: max-abs 2e-3 and relative L2 1e-3 against the oracle's
# float64 attention over the same dequantized cache.
ATOL = 2e-3
REL_L2 = 1e-3


def to_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device)


def gpu_prefill(w: W.Workload, K: np.ndarray, V: np.ndarray, max_seq=None) -> QuantizedKVCache:
    cache = QuantizedKVCache(config_from_workload(w, max_seq))
    cache.prefill(to_dev(K), to_dev(V))
    return cache


def oracle_row(w: W.Workload, k_bits: np.ndarray, v_bits: np.ndarray) -> KiviRow:
    row = KiviRow(w.head_dim, w.bits, w.group, w.residual, w.dtype)
    row.prefill(k_bits, v_bits)
    return row


def check_row_bits(cache: QuantizedKVCache, row_index: int, orow: KiviRow):
    """Packed records and the valid window slots must match byte for byte."""
    assert cache.quantized_len == orow.tq and cache.window_len == orow.r
    assert cache.window_head == orow.head
    ng = orow.tq // orow.G
    if ng:
        got = cache.records_view()[row_index, :ng].cpu().numpy()
        want = orow.records()
        if not np.array_equal(got, want):
            bad = np.argwhere(got != want)
            raise AssertionError(f"row {row_index}: {len(bad)} record bytes differ, first at {bad[:5].tolist()}")
    ring = cache.ring_view()[row_index].cpu().numpy().view(np.uint16)
    idx = (orow.head + np.arange(orow.r)) % orow.cap
    assert np.array_equal(ring[0][idx], orow.ring_k[idx]), f"row {row_index}: key window differs"
    assert np.array_equal(ring[1][idx], orow.ring_v[idx]), f"row {row_index}: value window differs"


def check_row_attention(out: np.ndarray, orow: KiviRow, q_bits: np.ndarray, w: W.Workload, scale=None):
    """out: float32 [g][d] from the GPU for one kv row; q_bits: [g][d]."""
    K, V = orow.dequantized()
    ref = oatt.attention(decode16(q_bits, w.dtype), K, V, w.scale if scale is None else scale)
    err = np.abs(out.astype(np.float64) - ref)
    rel = np.linalg.norm(out.astype(np.float64) - ref) / np.linalg.norm(ref)
    assert err.max() <= ATOL, f"max-abs {err.max():.3e} > {ATOL}"
    assert rel <= REL_L2, f"rel-L2 {rel:.3e} > {REL_L2}"
    return float(err.max()), float(rel)
