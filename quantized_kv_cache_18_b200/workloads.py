"""Seeded synthetic workloads for the quantized KV cache.

This module only draws random numbers and formats them as 16-bit inputs; it
holds none of the quantizer or attention arithmetic.  Both the CUDA path (via
the tests and the bench) and the float64 oracle are fed from it, so it imports
neither of them.

Shapes and value recipes follow the five workloads the KV-cache pages discuss:
a tiny KIVI case, a Llama-3-8B-shaped layer at 2 and 4 bits, a
Llama-3.1-70B-shaped 128K-token context, and a TurboQuant-style 3-bit case.
Keys carry per-channel outliers and values per-token outliers, the two
distributions the KIVI section of "Quantification du KV-Cache : TurboQuant et
l'etat de l'art en 2026" describes ("KIVI (2024)").

Every array is produced per (batch, kv-head) row from its own counter-derived
seed, so a test can regenerate any single row of a full-size workload without
drawing the rest.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Tuple

import numpy as np

# Stream tags: each random stream is keyed by (seed, tag, indices...).
_TAG_K, _TAG_V, _TAG_VOUT, _TAG_KCH, _TAG_Q, _TAG_STEP, _TAG_GAUSS = 1, 2, 3, 4, 5, 6, 7


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    scheme: str          # "kivi" or "turbo"
    batch: int
    num_kv_heads: int
    num_q_heads: int
    head_dim: int
    seq_len: int
    dtype: str           # "bf16" or "fp16"
    bits: int            # 2 / 4 (KIVI) or 3 (TurboQuant codes)
    group: int           # KIVI group size G; TurboQuant flush unit
    residual: int        # residual window R
    decode_steps: int = 1
    k_outlier_channels: Tuple[int, ...] = ()   # fixed channels (tiny); else drawn
    n_k_outlier_channels: int = 4
    k_outlier_scale: float = 20.0
    v_outlier_frac: float = 0.02
    v_outlier_scale: float = 10.0
    v_channel_outliers: bool = False          # TurboQuant: V gets the K channel recipe
    qjl_dim: int = 128
    rotation: str = "qr"                      # TurboQuant: "qr" (random orthogonal) or "wht"
    fp8_recent: bool = False                  # TurboQuant: FP8 window + anchors (mixed-format cache)
    anchor_tokens: int = 0
    seed: int = 0

    @property
    def gqa(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_seq(self) -> int:
        return self.seq_len + self.decode_steps

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


WORKLOADS: Dict[str, Workload] = {
    # 1 layer, batch 1, 2 KV heads, GQA 2, d 64, 512 tokens, fp16, G 32, R 32.
    "tiny": Workload("tiny", "kivi", 1, 2, 4, 64, 512, "fp16", 2, 32, 32,
                     k_outlier_channels=(3, 17), seed=0),
    # Llama-3-8B-shaped layer, 2-bit: 32 q heads, 8 kv heads, d 128, batch 16, 8192 tokens.
    "8b2": Workload("8b2", "kivi", 16, 8, 32, 128, 8192, "bf16", 2, 32, 128, seed=1),
    # Same shape at 4-bit, batch 64, 4096 tokens, G 64; 256 append+attend steps.
    "8b4": Workload("8b4", "kivi", 64, 8, 32, 128, 4096, "bf16", 4, 64, 128,
                    decode_steps=256, seed=2),
    # Llama-3.1-70B-shaped long context: 64 q heads, 8 kv heads, batch 1, 131072 tokens.
    "70b": Workload("70b", "kivi", 1, 8, 64, 128, 131072, "bf16", 2, 32, 128, seed=3),
    # TurboQuant-style 3-bit: 32 q heads, 8 kv heads, batch 8, 32768 tokens.
    "tq": Workload("tq", "turbo", 8, 8, 32, 128, 32768, "bf16", 3, 32, 128,
                   v_outlier_frac=0.0, v_channel_outliers=True, seed=4),
    # The same with the Walsh-Hadamard rotation H / sqrt(d) instead of the QR one.
    "tqw": Workload("tqw", "turbo", 8, 8, 32, 128, 32768, "bf16", 3, 32, 128,
                    v_outlier_frac=0.0, v_channel_outliers=True, rotation="wht", seed=4),
    # Mixed-format cache: the first 128 tokens and the window in FP8, the rest in TQ3.
    "tqm": Workload("tqm", "turbo", 8, 8, 32, 128, 32768, "bf16", 3, 32, 128,
                    v_outlier_frac=0.0, v_channel_outliers=True, fp8_recent=True, anchor_tokens=128, seed=4),
}


def with_sizes(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields changed (smaller parity cases)."""
    return dataclasses.replace(w, **kw)


# ---------------------------------------------------------------- 16-bit formatting
def round_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (inputs are finite)."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def round_to_fp16_bits(x32: np.ndarray) -> np.ndarray:
    return np.asarray(x32, dtype=np.float32).astype(np.float16).view(np.uint16)


def to_bits(x32: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return round_to_bf16_bits(x32)
    if dtype == "fp16":
        return round_to_fp16_bits(x32)
    raise ValueError(dtype)


def bits_to_float32(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Exact value of 16-bit patterns, widened to float32 (for display and torch)."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == "bf16":
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return bits.view(np.float16).astype(np.float32)


# ---------------------------------------------------------------- outlier choices
def k_outlier_channels(w: Workload) -> np.ndarray:
    """Key outlier channels: fixed for the tiny case, else drawn once per workload
    (shared by every batch row and head)."""
    if w.k_outlier_channels:
        return np.array(w.k_outlier_channels, dtype=np.int64)
    rng = np.random.default_rng([w.seed, _TAG_KCH])
    return np.sort(rng.choice(w.head_dim, size=w.n_k_outlier_channels, replace=False))


def v_outlier_tokens(w: Workload, b: int) -> np.ndarray:
    """Value outlier tokens of batch row b (shared across heads): a fixed count of
    round(frac * seq_len) prefill positions."""
    n = int(round(w.v_outlier_frac * w.seq_len))
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    rng = np.random.default_rng([w.seed, _TAG_VOUT, b])
    return np.sort(rng.choice(w.seq_len, size=n, replace=False))


# ---------------------------------------------------------------- generators
def prefill_row(w: Workload, b: int, h: int, seq_len: Optional[int] = None):
    """Keys and values of one (batch, kv-head) row: two uint16 arrays [S][d]."""
    S = w.seq_len if seq_len is None else seq_len
    d = w.head_dim
    rk = np.random.default_rng([w.seed, _TAG_K, b, h])
    rv = np.random.default_rng([w.seed, _TAG_V, b, h])
    k = rk.standard_normal((S, d), dtype=np.float32)
    v = rv.standard_normal((S, d), dtype=np.float32)
    ch = k_outlier_channels(w)
    k[:, ch] *= np.float32(w.k_outlier_scale)
    if w.v_channel_outliers:
        v[:, ch] *= np.float32(w.k_outlier_scale)
    vt = v_outlier_tokens(w, b)
    vt = vt[vt < S]
    v[vt, :] *= np.float32(w.v_outlier_scale)
    return to_bits(k, w.dtype), to_bits(v, w.dtype)


def prefill(w: Workload, rows=None, seq_len: Optional[int] = None):
    """Full prefill K and V as uint16 [B][Hkv][S][d] (or only the listed rows,
    as a dict {(b, h): (k, v)})."""
    S = w.seq_len if seq_len is None else seq_len
    if rows is not None:
        return {(b, h): prefill_row(w, b, h, S) for (b, h) in rows}
    K = np.empty((w.batch, w.num_kv_heads, S, w.head_dim), dtype=np.uint16)
    V = np.empty_like(K)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            K[b, h], V[b, h] = prefill_row(w, b, h, S)
    return K, V


def query(w: Workload, step: int = 0) -> np.ndarray:
    """Decode query of a step: uint16 [B][Hq][d], N(0, 1)."""
    r = np.random.default_rng([w.seed, _TAG_Q, step])
    q = r.standard_normal((w.batch, w.num_q_heads, w.head_dim), dtype=np.float32)
    return to_bits(q, w.dtype)


def decode_token(w: Workload, step: int):
    """New key and value of decode step `step` (1-based): uint16 [B][Hkv][d] each.
    Keys keep the outlier channels; a value row is an outlier token with
    probability v_outlier_frac (drawn per batch row, shared across heads)."""
    r = np.random.default_rng([w.seed, _TAG_STEP, step])
    shape = (w.batch, w.num_kv_heads, w.head_dim)
    k = r.standard_normal(shape, dtype=np.float32)
    v = r.standard_normal(shape, dtype=np.float32)
    ch = k_outlier_channels(w)
    k[:, :, ch] *= np.float32(w.k_outlier_scale)
    if w.v_channel_outliers:
        v[:, :, ch] *= np.float32(w.k_outlier_scale)
    hit = r.random(w.batch) < w.v_outlier_frac
    v[hit] *= np.float32(w.v_outlier_scale)
    return to_bits(k, w.dtype), to_bits(v, w.dtype)


def gaussian_matrix(w: Workload, tag: str, rows: int, cols: int) -> np.ndarray:
    """Seeded N(0, 1) matrix drawn in float64 and stored as float32: the random
    draw behind the TurboQuant rotation ("rot") and the QJL projection ("qjl")."""
    t = {"rot": 0, "qjl": 1}[tag]
    r = np.random.default_rng([w.seed, _TAG_GAUSS, t])
    return r.standard_normal((rows, cols)).astype(np.float32)
