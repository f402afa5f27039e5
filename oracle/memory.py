"""Byte accounting of the KV cache.  Test infrastructure only.

* Memory formula ("Quantification du KV-Cache : TurboQuant et l'etat de l'art
  en 2026", section "Le probleme : le KV-cache, gouffre silencieux"):
  bytes = 2 * L * H * d * S * bytes_per_element, the 2 counting keys and values.
* Packing ratios (same page, "TurboQuant : les cinq innovations" item 3): codes
  alone take 16 / b times less than fp16, i.e. /4 at INT4 and /8 at INT2.
"""
from __future__ import annotations


def kv_cache_bytes(layers: int, kv_heads: int, head_dim: int, seq_len: int, bytes_per_elem: float) -> float:
    return 2 * layers * kv_heads * head_dim * seq_len * bytes_per_elem


def codes_only_ratio(bits: int, ref_bits: int = 16) -> float:
    return ref_bits / bits


def kivi_bytes_per_token(head_dim: int, bits: int, group: int) -> float:
    """Packed bytes of one quantized token of one kv head: key and value codes,
    the key (scale, zero) fp16 pair per channel shared by a group of G tokens,
    and the value (scale, zero) fp16 pair of the token."""
    codes = 2 * head_dim * bits / 8
    key_meta = head_dim * 2 * 2 / group
    value_meta = 2 * 2
    return codes + key_meta + value_meta


def window_bytes_per_token(head_dim: int) -> int:
    """A window token keeps its 16-bit key and value."""
    return 2 * head_dim * 2


def kivi_cache_bytes(batch, kv_heads, head_dim, bits, group, tq, r) -> float:
    """Bytes one decode step reads: every quantized token plus every window token."""
    return batch * kv_heads * (tq * kivi_bytes_per_token(head_dim, bits, group)
                               + r * window_bytes_per_token(head_dim))
