"""Single-token decode attention, float64.  Test infrastructure only.

Decode reads the whole cache for every new token ("La compression du cache KV
est une decision d'infrastructure...", section "... quand la HBM, pas les
FLOPs, est votre plafond"); each new token "looks back" at the stored keys and
values ("Quantification du KV-Cache ...", "Le probleme").  The output of query
head h is softmax(scale * q_h . k_t) weighted values over every cached token t,
the quantized ones dequantized and the window ones exact, with query head h
reading kv head h // (Hq / Hkv).

Partial states over disjoint token ranges are merged with a log-sum-exp that
normalises globally, as Minima-KV does for its per-format partial attention
("KV-cache compresse et modeles 4-bit ...", section "Minima-KV : la
compression sans eviction").
"""
from __future__ import annotations

import math

import numpy as np


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """q [g][d], K/V [T][d] -> [g][d]; one matmul per side, float64."""
    s = scale * (np.asarray(q, np.float64) @ np.asarray(K, np.float64).T)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    return (p @ np.asarray(V, np.float64)) / p.sum(axis=1, keepdims=True)


def attention_loops(q, K, V, scale) -> list:
    """The same, as textbook loops in pure Python (small inputs only)."""
    out = []
    for qh in q:
        scores = [scale * sum(float(a) * float(b) for a, b in zip(qh, k)) for k in K]
        mx = max(scores)
        w = [math.exp(x - mx) for x in scores]
        tot = sum(w)
        out.append([sum(w[t] * float(V[t][c]) for t in range(len(V))) / tot for c in range(len(V[0]))])
    return out


def partial(q, K, V, scale):
    """(m [g], l [g], o [g][d]) over one token range; o is already divided by l."""
    s = scale * (np.asarray(q, np.float64) @ np.asarray(K, np.float64).T)
    m = s.max(axis=1)
    p = np.exp(s - m[:, None])
    l = p.sum(axis=1)
    return m, l, (p @ np.asarray(V, np.float64)) / l[:, None]


def merge(parts) -> np.ndarray:
    """Combine partials of disjoint ranges: M = max m_j, L = sum l_j e^(m_j - M),
    out = sum l_j e^(m_j - M) o_j / L."""
    M = np.max([m for m, _, _ in parts], axis=0)
    w = [l * np.exp(m - M) for m, l, _ in parts]
    L = np.sum(w, axis=0)
    return np.sum([wj[:, None] * o for wj, (_, _, o) in zip(w, parts)], axis=0) / L[:, None]


def gqa_attention(q_heads: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """Query heads [g][d] of one kv head against that head's cache."""
    return attention(q_heads, K, V, scale)
