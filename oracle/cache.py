"""One (batch, kv-head) row of the quantized KV cache, float64.  Test
infrastructure only.

Residual window ("Quantification du KV-Cache : TurboQuant et l'etat de l'art en
2026", "TurboQuant : les cinq innovations" item 4 "Fenetre residuelle"; and
section "KIVI (2024)", "un residu FP16 pour les derniers tokens"): the most
recent tokens stay unquantized and the attention kernel sees the hybrid cache
as one sequence.  The pages give the window size (128) but not how tokens move
out of it.  Reading used here:

* prefill of S tokens quantizes T_q = G * floor(max(0, S - R) / G) tokens and
  keeps r = S - T_q in the window (R <= r < R + G once S >= R);
* each appended token goes into the window; when r reaches R + G the oldest G
  window tokens are quantized as one new key group and G value tokens
  (T_q += G, r -= G), so key groups are always whole and the last R tokens
  are always exact;
* the window stores the 16-bit inputs unchanged (bf16 stays bf16): "FP16" on
  the pages is read as "16-bit, not quantized".

The window lives in a ring of R + G slots: logical window token i sits in slot
(head + i) mod (R + G); a flush advances head by G.
"""
from __future__ import annotations

import numpy as np

from . import kivi
from .layout import pack_records
from .numerics import decode16


def quantized_len(S: int, R: int, G: int) -> int:
    """T_q after a prefill of S tokens."""
    return G * (max(0, S - R) // G)


class KiviRow:
    def __init__(self, d: int, bits: int, G: int, R: int, dtype: str):
        assert R % G == 0
        self.d, self.bits, self.G, self.R, self.dtype = d, bits, G, R, dtype
        self.cap = R + G
        self.kc = np.zeros((0, d), np.uint8)
        self.vc = np.zeros((0, d), np.uint8)
        self.ks = np.zeros((0, d))
        self.kz = np.zeros((0, d))
        self.vs = np.zeros(0)
        self.vz = np.zeros(0)
        self.ring_k = np.zeros((self.cap, d), np.uint16)
        self.ring_v = np.zeros((self.cap, d), np.uint16)
        self.head = 0
        self.r = 0
        self.ok = True          # False once a range condition was hit

    # ------------------------------------------------------------ state
    @property
    def tq(self) -> int:
        return self.kc.shape[0]

    @property
    def seq_len(self) -> int:
        return self.tq + self.r

    def window_bits(self):
        idx = (self.head + np.arange(self.r)) % self.cap
        return self.ring_k[idx], self.ring_v[idx]

    # ------------------------------------------------------------ quantization
    def _quantize_tokens(self, kb: np.ndarray, vb: np.ndarray):
        """Quantize whole groups of tokens (16-bit patterns [n*G][d]) and append
        them to the quantized part."""
        G, bits = self.G, self.bits
        k = decode16(kb, self.dtype)
        v = decode16(vb, self.dtype)
        c, s, z = kivi.quantize_key_groups(k, bits, G)
        self.ok &= kivi.in_range(k, s, z)
        self.kc = np.concatenate([self.kc, c])
        self.ks = np.concatenate([self.ks, s])
        self.kz = np.concatenate([self.kz, z])
        c, s, z = kivi.quantize_values(v, bits)
        self.ok &= kivi.in_range(v, s, z)
        self.vc = np.concatenate([self.vc, c])
        self.vs = np.concatenate([self.vs, s])
        self.vz = np.concatenate([self.vz, z])

    def prefill(self, kb: np.ndarray, vb: np.ndarray):
        """kb, vb: uint16 [S][d]."""
        assert self.seq_len == 0
        S = kb.shape[0]
        tq = quantized_len(S, self.R, self.G)
        if tq:
            self._quantize_tokens(kb[:tq], vb[:tq])
        self.r = S - tq
        self.head = 0
        self.ring_k[:self.r] = kb[tq:]
        self.ring_v[:self.r] = vb[tq:]

    def append(self, kb: np.ndarray, vb: np.ndarray):
        """One new token: kb, vb uint16 [d]."""
        slot = (self.head + self.r) % self.cap
        self.ring_k[slot] = kb
        self.ring_v[slot] = vb
        self.r += 1
        if self.r == self.R + self.G:
            idx = (self.head + np.arange(self.G)) % self.cap
            self._quantize_tokens(self.ring_k[idx], self.ring_v[idx])
            self.head = (self.head + self.G) % self.cap
            self.r -= self.G

    # ------------------------------------------------------------ views
    def dequantized(self):
        """Logical cache as float64 [T_q + r][d] keys and values: the dequantized
        tokens in order, then the window tokens in order."""
        kq = kivi.dequant(self.kc, np.repeat(self.ks, self.G, axis=0), np.repeat(self.kz, self.G, axis=0))
        vq = kivi.dequant(self.vc, self.vs[:, None], self.vz[:, None])
        wk, wv = self.window_bits()
        return (np.concatenate([kq, decode16(wk, self.dtype)]),
                np.concatenate([vq, decode16(wv, self.dtype)]))

    def records(self) -> np.ndarray:
        assert self.G % 32 == 0
        return pack_records(self.kc, self.ks, self.kz, self.vc, self.vs, self.vz,
                            self.d, self.bits, self.G)
