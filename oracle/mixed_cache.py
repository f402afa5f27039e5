"""One (batch, kv-head) row of the mixed-format cache, float64.  Test
infrastructure only.

Minima-KV keeps recent and protected ("Anchor") pages in FP8, moves older
pages to TQ3, and merges the attention over all of them with one globally
normalised online softmax ("KV-cache compresse et modeles 4-bit ...", section
"Minima-KV : la compression sans eviction").  Readings where the page is
silent:
* anchors are the first A tokens of the sequence (A a multiple of 32), taken
  from the prefill and kept in FP8 for good;
* the recent window works as in the TurboQuant cache (at least R tokens, G =
  32 leave it at a time), its tokens stored in FP8 (oracle/fp8.py);
* tokens leaving the window are quantized to TQ3 from their FP8 values (the
  page ages from FP8 into TQ3; the 16-bit originals are gone by then);
* prefill: tokens [0, A) are anchors, the next T_q = 32 floor(max(0, S - A -
  R) / 32) are quantized to TQ3 from the 16-bit inputs, the rest enter the
  window; S >= A.
Token row format (144 bytes): 128 E4M3 codes, the fp16 scale, 14 zero bytes.
"""
from __future__ import annotations

import numpy as np

from . import fp8, turbo
from .numerics import decode16, fp16_bits
from .turbo_cache import pack_tbs

ROW_BYTES = 144


def pack_fp8_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """[T][d] codes and [T] scales -> [T][ROW_BYTES] uint8 token rows."""
    t, d = codes.shape
    out = np.zeros((t, ROW_BYTES), np.uint8)
    out[:, :d] = codes
    out[:, d:d + 2] = fp16_bits(scales).view(np.uint8).reshape(t, 2)
    return out


class MixedRow:
    def __init__(self, d: int, R: int, A: int, dtype: str, Pi: np.ndarray, S: np.ndarray, levels: np.ndarray,
                 thresholds: np.ndarray, G: int = 32):
        assert R % G == 0 and A % 32 == 0
        self.d, self.R, self.A, self.G, self.dtype = d, R, A, G, dtype
        self.Pi, self.S, self.levels, self.thresholds = Pi, S, levels, thresholds
        self.cap = R + G
        self.kq = {"codes": np.zeros((0, d), np.uint8), "n": np.zeros(0), "gamma": np.zeros(0),
                   "signs": np.zeros((0, S.shape[0]), np.uint8), "y": np.zeros((0, d)),
                   "se": np.zeros((0, S.shape[0]))}
        self.vq = {"codes": np.zeros((0, d), np.uint8), "n": np.zeros(0), "y": np.zeros((0, d))}
        # FP8 rows: anchors [A], window ring [cap]; codes and scales
        self.anc = {kv: (np.zeros((A, d), np.uint8), np.zeros(A)) for kv in "kv"}
        self.ring = {kv: (np.zeros((self.cap, d), np.uint8), np.zeros(self.cap)) for kv in "kv"}
        self.head = 0
        self.r = 0
        self.k_in = np.zeros((0, d))   # the float64 vectors that went into TQ3, in order
        self.v_in = np.zeros((0, d))

    @property
    def tq(self) -> int:
        return self.kq["codes"].shape[0]

    def _quantize(self, k: np.ndarray, v: np.ndarray):
        self.k_in = np.concatenate([self.k_in, k])
        self.v_in = np.concatenate([self.v_in, v])
        a = turbo.quantize(k, self.Pi, self.levels, self.thresholds, self.S)
        b = turbo.quantize(v, self.Pi, self.levels, self.thresholds)
        for key in ("codes", "n", "gamma", "signs", "y", "se"):
            self.kq[key] = np.concatenate([self.kq[key], a[key]])
        for key in ("codes", "n", "y"):
            self.vq[key] = np.concatenate([self.vq[key], b[key]])

    def prefill(self, kb, vb):
        S = kb.shape[0]
        assert S >= self.A
        k, v = decode16(kb, self.dtype), decode16(vb, self.dtype)
        for kv, x in (("k", k), ("v", v)):
            self.anc[kv] = fp8.fp8_rows(x[:self.A])
        rest = S - self.A
        tq = self.G * (max(0, rest - self.R) // self.G)
        if tq:
            self._quantize(k[self.A:self.A + tq], v[self.A:self.A + tq])
        self.r = rest - tq
        self.head = 0
        for kv, x in (("k", k), ("v", v)):
            c, s = fp8.fp8_rows(x[self.A + tq:])
            self.ring[kv][0][:self.r], self.ring[kv][1][:self.r] = c, s

    def append(self, kb, vb):
        slot = (self.head + self.r) % self.cap
        for kv, x in (("k", kb), ("v", vb)):
            c, s = fp8.fp8_rows(decode16(np.asarray(kb if kv == "k" else vb)[None], self.dtype))
            self.ring[kv][0][slot], self.ring[kv][1][slot] = c[0], s[0]
        self.r += 1
        if self.r == self.R + self.G:
            idx = (self.head + np.arange(self.G)) % self.cap
            self._quantize(fp8.fp8_dequant(self.ring["k"][0][idx], self.ring["k"][1][idx]),
                           fp8.fp8_dequant(self.ring["v"][0][idx], self.ring["v"][1][idx]))
            self.head = (self.head + self.G) % self.cap
            self.r -= self.G

    def window_idx(self):
        return (self.head + np.arange(self.r)) % self.cap

    def fp8_values(self, kv: str) -> np.ndarray:
        """Dequantized anchors followed by the window, [A + r][d]."""
        idx = self.window_idx()
        c, s = self.ring[kv]
        return np.concatenate([fp8.fp8_dequant(*self.anc[kv]), fp8.fp8_dequant(c[idx], s[idx])])

    def attention(self, q_bits: np.ndarray, scale: float) -> np.ndarray:
        q = decode16(q_bits, self.dtype)
        return turbo.attention(q, self.Pi, self.S, self.levels, self.kq, self.vq, self.fp8_values("k"),
                               self.fp8_values("v"), scale)

    def records(self) -> np.ndarray:
        return pack_tbs(self.kq["codes"], self.kq["n"], self.kq["gamma"], self.kq["signs"],
                        self.vq["codes"], self.vq["n"], self.d, self.S.shape[0])

    def anchor_rows(self, kv: str) -> np.ndarray:
        return pack_fp8_rows(*self.anc[kv])

    def ring_rows(self, kv: str) -> np.ndarray:
        return pack_fp8_rows(*self.ring[kv])
