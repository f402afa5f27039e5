"""One (batch, kv-head) row of the TurboQuant-style cache and its packed form
(format v1).  Test infrastructure only.

The window works as for the KIVI cache (oracle/cache.py): R most recent tokens
at least stay unquantized in a ring of R + G slots, and G = 32 tokens leave it
at a time; here G is only the flush unit, there are no groups.

Packed token block (TB, 32 tokens of one row), 4032 bytes:
  [key codes 1664][value codes 1664][key sign bits 512][key meta 128][value meta 64]
Codes.  Two 3-bit codes of a fragment pair form a 6-bit index lo + 8 hi; five
indices fill a 32-bit word (bits 6f .. 6f+5, bits 30-31 zero).  A lane owns 64
pairs per TB in slots 0..63 (word slot // 5, field slot % 5) stored as words
0..11 in three 16-byte pieces at byte 16 (32 p + lane) and word 12 at byte
1536 + 4 lane.
  key pair (nt, kt, rho) of lane (gr, tc): token 8nt+gr, coordinates
      16kt+8rho+2tc (lo) and +1 (hi); slot = 16 nt + 2 kt + rho
  value pair (kt, nt, rho): coordinate 8nt+gr, tokens 16kt+8rho+2tc (lo) and +1
      (hi); slot = 32 kt + 2 nt + rho
Sign bits.  Key pair (nt, kt, rho) of lane (gr, tc): token 8nt+gr, sketch rows
16kt+8rho+2tc (lo) and +1 (hi); slot = 16 nt + 2 kt + rho, word slot // 16 of
the lane (16-byte piece at byte 16 lane), lo bit at slot % 16, hi bit at
16 + slot % 16.
Meta.  Token t = 16kt+8rho+2tc+e of the TB at entry 8tc+4kt+2rho+e: keys as
(fp16 n, fp16 gamma) pairs, values as fp16 n.
"""
from __future__ import annotations

import functools

import numpy as np

from . import turbo
from .numerics import decode16, fp16_bits

TB_BYTES = 4032
CODE_BYTES = 1664
SIGN_BYTES = 512


def _code_word_offset(lane: int, w: int) -> int:
    return 16 * (32 * (w >> 2) + lane) + 4 * (w & 3) if w < 12 else 1536 + 4 * lane


@functools.lru_cache(maxsize=None)
def key_code_map(d: int = 128):
    """[32 tokens][d] -> (byte offset of the word, bit offset of the 3-bit code)."""
    off = np.full((32, d), -1, np.int64)
    bit = np.full((32, d), -1, np.int64)
    for lane in range(32):
        gr, tc = lane >> 2, lane & 3
        for nt in range(4):
            for kt in range(d // 16):
                for rho in range(2):
                    slot = 16 * nt + 2 * kt + rho
                    w, f = divmod(slot, 5)
                    for e in range(2):
                        t, c = 8 * nt + gr, 16 * kt + 8 * rho + 2 * tc + e
                        off[t, c] = _code_word_offset(lane, w)
                        bit[t, c] = 6 * f + 3 * e
    assert (off >= 0).all()
    return off, bit


@functools.lru_cache(maxsize=None)
def value_code_map(d: int = 128):
    off = np.full((32, d), -1, np.int64)
    bit = np.full((32, d), -1, np.int64)
    for lane in range(32):
        gr, tc = lane >> 2, lane & 3
        for kt in range(2):
            for nt in range(d // 8):
                for rho in range(2):
                    slot = 32 * kt + 2 * nt + rho
                    w, f = divmod(slot, 5)
                    for e in range(2):
                        t, c = 16 * kt + 8 * rho + 2 * tc + e, 8 * nt + gr
                        off[t, c] = _code_word_offset(lane, w)
                        bit[t, c] = 6 * f + 3 * e
    assert (off >= 0).all()
    return off, bit


@functools.lru_cache(maxsize=None)
def sign_map(m: int = 128):
    """[32 tokens][m] -> (byte offset of the word, bit)."""
    off = np.full((32, m), -1, np.int64)
    bit = np.full((32, m), -1, np.int64)
    for lane in range(32):
        gr, tc = lane >> 2, lane & 3
        for nt in range(4):
            for kt in range(m // 16):
                for rho in range(2):
                    slot = 16 * nt + 2 * kt + rho
                    w, q = divmod(slot, 16)
                    for e in range(2):
                        t, i = 8 * nt + gr, 16 * kt + 8 * rho + 2 * tc + e
                        off[t, i] = 16 * lane + 4 * w
                        bit[t, i] = q + 16 * e
    assert (off >= 0).all()
    return off, bit


@functools.lru_cache(maxsize=None)
def meta_perm():
    pos = np.full(32, -1, np.int64)
    for tc in range(4):
        for kt in range(2):
            for rho in range(2):
                for e in range(2):
                    pos[16 * kt + 8 * rho + 2 * tc + e] = 8 * tc + 4 * kt + 2 * rho + e
    return pos


def _scatter(vals: np.ndarray, off: np.ndarray, bit: np.ndarray, nbytes: int) -> np.ndarray:
    """vals [n_tb][32][k] small ints -> bytes [n_tb][nbytes] (disjoint bit fields)."""
    n = vals.shape[0]
    words = np.zeros((n, nbytes // 4), np.uint64)
    widx = (off // 4).reshape(-1)
    contrib = vals.reshape(n, -1).astype(np.uint64) << bit.reshape(-1).astype(np.uint64)
    for i in range(n):
        np.add.at(words[i], widx, contrib[i])
    return np.ascontiguousarray(words.astype(np.uint32)).view(np.uint8).reshape(n, nbytes)


def _gather(blocks: np.ndarray, off: np.ndarray, bit: np.ndarray, width: int) -> np.ndarray:
    n = blocks.shape[0]
    words = np.ascontiguousarray(blocks).view(np.uint32).reshape(n, -1)
    w = words[:, (off // 4).reshape(-1)]
    v = (w >> bit.reshape(-1).astype(np.uint32)) & np.uint32((1 << width) - 1)
    return v.reshape(n, 32, -1).astype(np.uint8)


def pack_tbs(kc, kn, kg, ks, vc, vn, d: int = 128, m: int = 128) -> np.ndarray:
    """Quantized tokens of one row (T a multiple of 32) -> uint8 [T/32][TB_BYTES].
    kc, vc: codes [T][d]; kn, kg, vn: fp16 values [T]; ks: sign bits [T][m]."""
    T = kc.shape[0]
    n_tb = T // 32
    ko, kb = key_code_map(d)
    vo, vb = value_code_map(d)
    so, sb = sign_map(m)
    kblk = _scatter(kc.reshape(n_tb, 32, d), ko, kb, CODE_BYTES)
    vblk = _scatter(vc.reshape(n_tb, 32, d), vo, vb, CODE_BYTES)
    sblk = _scatter(ks.reshape(n_tb, 32, m), so, sb, SIGN_BYTES)
    perm = meta_perm()
    km = np.zeros((n_tb, 32), np.uint32)
    km[:, perm] = (fp16_bits(kn).reshape(n_tb, 32).astype(np.uint32)
                   | (fp16_bits(kg).reshape(n_tb, 32).astype(np.uint32) << np.uint32(16)))
    vm = np.zeros((n_tb, 32), np.uint16)
    vm[:, perm] = fp16_bits(vn).reshape(n_tb, 32)
    rec = np.concatenate([kblk, vblk, sblk, np.ascontiguousarray(km).view(np.uint8),
                          np.ascontiguousarray(vm).view(np.uint8)], axis=1)
    assert rec.shape[1] == TB_BYTES
    return rec


def unpack_tbs(rec: np.ndarray, d: int = 128, m: int = 128):
    n_tb = rec.shape[0]
    ko, kb = key_code_map(d)
    vo, vb = value_code_map(d)
    so, sb = sign_map(m)
    o = 0
    kc = _gather(rec[:, o:o + CODE_BYTES], ko, kb, 3).reshape(-1, d); o += CODE_BYTES
    vc = _gather(rec[:, o:o + CODE_BYTES], vo, vb, 3).reshape(-1, d); o += CODE_BYTES
    ks = _gather(rec[:, o:o + SIGN_BYTES], so, sb, 1).reshape(-1, m); o += SIGN_BYTES
    perm = meta_perm()
    km = np.ascontiguousarray(rec[:, o:o + 128]).view(np.uint32)[:, perm]; o += 128
    vm = np.ascontiguousarray(rec[:, o:o + 64]).view(np.uint16)[:, perm]
    kn = (km & np.uint32(0xFFFF)).astype(np.uint16).view(np.float16).astype(np.float64).reshape(-1)
    kg = (km >> np.uint32(16)).astype(np.uint16).view(np.float16).astype(np.float64).reshape(-1)
    vn = vm.view(np.float16).astype(np.float64).reshape(-1)
    return kc, kn, kg, ks, vc, vn


class TurboRow:
    """Prefill / append / attention of one row with TurboQuant-quantized tokens
    and the exact 16-bit window."""

    def __init__(self, d: int, R: int, dtype: str, Pi: np.ndarray, S: np.ndarray, levels: np.ndarray,
                 thresholds: np.ndarray, G: int = 32):
        assert R % G == 0
        self.d, self.R, self.G, self.dtype = d, R, G, dtype
        self.Pi, self.S, self.levels, self.thresholds = Pi, S, levels, thresholds
        self.cap = R + G
        self.kq = {"codes": np.zeros((0, d), np.uint8), "n": np.zeros(0), "gamma": np.zeros(0),
                   "signs": np.zeros((0, S.shape[0]), np.uint8), "y": np.zeros((0, d)), "se": np.zeros((0, S.shape[0]))}
        self.vq = {"codes": np.zeros((0, d), np.uint8), "n": np.zeros(0), "y": np.zeros((0, d))}
        self.ring_k = np.zeros((self.cap, d), np.uint16)
        self.ring_v = np.zeros((self.cap, d), np.uint16)
        self.head = 0
        self.r = 0

    @property
    def tq(self) -> int:
        return self.kq["codes"].shape[0]

    def _quantize(self, kb, vb):
        k = decode16(kb, self.dtype)
        v = decode16(vb, self.dtype)
        a = turbo.quantize(k, self.Pi, self.levels, self.thresholds, self.S)
        b = turbo.quantize(v, self.Pi, self.levels, self.thresholds)
        for key in ("codes", "n", "gamma", "signs", "y", "se"):
            self.kq[key] = np.concatenate([self.kq[key], a[key]])
        for key in ("codes", "n", "y"):
            self.vq[key] = np.concatenate([self.vq[key], b[key]])

    def prefill(self, kb, vb):
        S = kb.shape[0]
        tq = self.G * (max(0, S - self.R) // self.G)
        if tq:
            self._quantize(kb[:tq], vb[:tq])
        self.r = S - tq
        self.head = 0
        self.ring_k[:self.r] = kb[tq:]
        self.ring_v[:self.r] = vb[tq:]

    def append(self, kb, vb):
        slot = (self.head + self.r) % self.cap
        self.ring_k[slot] = kb
        self.ring_v[slot] = vb
        self.r += 1
        if self.r == self.R + self.G:
            idx = (self.head + np.arange(self.G)) % self.cap
            self._quantize(self.ring_k[idx], self.ring_v[idx])
            self.head = (self.head + self.G) % self.cap
            self.r -= self.G

    def window_bits(self):
        idx = (self.head + np.arange(self.r)) % self.cap
        return self.ring_k[idx], self.ring_v[idx]

    def attention(self, q_bits: np.ndarray, scale: float) -> np.ndarray:
        wk, wv = self.window_bits()
        q = decode16(q_bits, self.dtype)
        return turbo.attention(q, self.Pi, self.S, self.levels, self.kq, self.vq,
                               decode16(wk, self.dtype), decode16(wv, self.dtype), scale)

    def records(self) -> np.ndarray:
        return pack_tbs(self.kq["codes"], self.kq["n"], self.kq["gamma"], self.kq["signs"],
                        self.vq["codes"], self.vq["n"], self.d, self.S.shape[0])
