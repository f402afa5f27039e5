"""Packed cache layout (format v1), written out independently of the CUDA code.
Test infrastructure only.

The pages fix the packing density -- 16 INT2 or 8 INT4 codes per 32-bit word,
dequantized in registers ("Quantification du KV-Cache : TurboQuant et l'etat de
l'art en 2026", "TurboQuant : les cinq innovations", item 3 "Bit-packing
dense") -- but not the order of codes inside the words.  Format v1 orders them
for the decode kernel's tensor-core fragments; the order is a bijection, so it
changes no value, only where a code sits.

Notation: a token block (TB) is 32 consecutive tokens; lane L in [0, 32) has
gr = L >> 2 and tc = L & 3; every lane owns P = d*b/32 words of a TB's key
codes and P words of its value codes.

Key codes of a TB.  Pair (nt, kt, rho) of lane (gr, tc) holds the codes of
token 8 nt + gr at channels c0 = 16 kt + 8 rho + 2 tc (low half-word) and c0+1
(high half-word); u = 2 kt + rho.
  2-bit: j' = u & 3, slot = nt*(d/32) + (u >> 2), word = slot >> 1, j = 4(slot & 1) + j'
  4-bit: j' = u & 1, slot = nt*(d/16) + (u >> 1), word = slot >> 1, j = 2(slot & 1) + j'
Value codes of a TB.  Pair (kt, nt, rho) of lane (gr, tc) holds the codes of
channel 8 nt + gr at tokens t0 = 16 kt + 8 rho + 2 tc (low) and t0+1 (high);
u = 2 kt + rho.
  2-bit: j' = u,     slot = nt,                 word = slot >> 1, j = 4(slot & 1) + j'
  4-bit: j' = u & 1, slot = 2 nt + (u >> 1),    word = slot >> 1, j = 2(slot & 1) + j'
In a word, the low code of pair j sits at bit b*j and the high code at bit
16 + b*j.  Word w of lane L is stored at byte 16*(32*(w >> 2) + L) + 4*(w & 3)
of the TB's code block, so a warp reads a block as 16-byte pieces, one per lane.

Key metadata of a group: d fp16 scales then d fp16 zeros, channel
c = 16 kt + 8 rho + 2 tc + e stored at position
8 (4 (kt >> 1) + tc) + 4 (kt & 1) + 2 rho + e, so the lanes of one tc read 16
consecutive bytes per k-tile pair and the four tc read adjacent chunks.
Value metadata of a TB: 32 entries of 4 bytes (fp16 scale in the low half,
fp16 zero in the high half); token t = 16 kt + 8 rho + 2 tc + e stored at
entry 8 tc + 4 kt + 2 rho + e.

Group record (G tokens, G a multiple of 32): key codes of TBs 0..G/32-1, value
codes of TBs 0..G/32-1, key scales, key zeros, value metadata of TBs 0..G/32-1.
Size: G*d*b/4 + 4 d + 4 G bytes (2688 B for 2-bit, d 128, G 32).
"""
from __future__ import annotations

import functools

import numpy as np

from .numerics import fp16_bits


def record_bytes(d: int, bits: int, G: int) -> int:
    return G * d * bits // 4 + 4 * d + 4 * G


def tb_code_bytes(d: int, bits: int) -> int:
    return 32 * d * bits // 8


def _word_byte_offset(lane: int, w: int) -> int:
    return 16 * (32 * (w >> 2) + lane) + 4 * (w & 3)


@functools.lru_cache(maxsize=None)
def key_code_map(d: int, bits: int):
    """For a key TB: arrays [32 tokens][d channels] of (byte offset of the word,
    bit offset inside the word) where that code lives."""
    off = np.full((32, d), -1, dtype=np.int64)
    bit = np.full((32, d), -1, dtype=np.int64)
    for lane in range(32):
        gr, tc = lane >> 2, lane & 3
        for nt in range(4):
            for kt in range(d // 16):
                for rho in range(2):
                    u = 2 * kt + rho
                    if bits == 2:
                        jp, slot = u & 3, nt * (d // 32) + (u >> 2)
                        j = 4 * (slot & 1) + jp
                    else:
                        jp, slot = u & 1, nt * (d // 16) + (u >> 1)
                        j = 2 * (slot & 1) + jp
                    w = slot >> 1
                    for e in range(2):
                        t, c = 8 * nt + gr, 16 * kt + 8 * rho + 2 * tc + e
                        assert off[t, c] < 0
                        off[t, c] = _word_byte_offset(lane, w)
                        bit[t, c] = bits * j + 16 * e
    assert (off >= 0).all()
    return off, bit


@functools.lru_cache(maxsize=None)
def value_code_map(d: int, bits: int):
    """Same for a value TB: [32 tokens][d channels] -> (byte offset, bit offset)."""
    off = np.full((32, d), -1, dtype=np.int64)
    bit = np.full((32, d), -1, dtype=np.int64)
    for lane in range(32):
        gr, tc = lane >> 2, lane & 3
        for kt in range(2):
            for nt in range(d // 8):
                for rho in range(2):
                    u = 2 * kt + rho
                    if bits == 2:
                        jp, slot = u, nt
                        j = 4 * (slot & 1) + jp
                    else:
                        jp, slot = u & 1, 2 * nt + (u >> 1)
                        j = 2 * (slot & 1) + jp
                    w = slot >> 1
                    for e in range(2):
                        t, c = 16 * kt + 8 * rho + 2 * tc + e, 8 * nt + gr
                        assert off[t, c] < 0
                        off[t, c] = _word_byte_offset(lane, w)
                        bit[t, c] = bits * j + 16 * e
    assert (off >= 0).all()
    return off, bit


@functools.lru_cache(maxsize=None)
def key_meta_perm(d: int) -> np.ndarray:
    """position[c] of channel c in the key scale (and zero) arrays."""
    pos = np.full(d, -1, dtype=np.int64)
    for tc in range(4):
        for kt in range(d // 16):
            for rho in range(2):
                for e in range(2):
                    pos[16 * kt + 8 * rho + 2 * tc + e] = 8 * (4 * (kt >> 1) + tc) + 4 * (kt & 1) + 2 * rho + e
    assert sorted(pos.tolist()) == list(range(d))
    return pos


@functools.lru_cache(maxsize=None)
def value_meta_perm() -> np.ndarray:
    """entry[t] of token t (0..31) in a TB's value metadata."""
    pos = np.full(32, -1, dtype=np.int64)
    for tc in range(4):
        for kt in range(2):
            for rho in range(2):
                for e in range(2):
                    pos[16 * kt + 8 * rho + 2 * tc + e] = 8 * tc + 4 * kt + 2 * rho + e
    assert sorted(pos.tolist()) == list(range(32))
    return pos


def _pack_tbs(codes: np.ndarray, off: np.ndarray, bit: np.ndarray, nbytes: int) -> np.ndarray:
    """codes [n_tb][32][d] -> bytes [n_tb][nbytes] via the (off, bit) map."""
    n = codes.shape[0]
    nwords = nbytes // 4
    widx = (off // 4).reshape(-1)
    order = np.argsort(widx, kind="stable")
    per_word = widx.size // nwords
    assert np.array_equal(widx[order].reshape(nwords, per_word),
                          np.repeat(np.arange(nwords), per_word).reshape(nwords, per_word))
    contrib = codes.reshape(n, -1).astype(np.uint64) << bit.reshape(-1).astype(np.uint64)
    # every word receives exactly per_word disjoint bit fields: their sum is their OR
    words = contrib[:, order].reshape(n, nwords, per_word).sum(axis=2)
    return np.ascontiguousarray(words.astype(np.uint32)).view(np.uint8).reshape(n, nbytes)


def _unpack_tbs(blocks: np.ndarray, off: np.ndarray, bit: np.ndarray, bits: int) -> np.ndarray:
    n = blocks.shape[0]
    words = np.ascontiguousarray(blocks).view(np.uint32).reshape(n, -1)
    w = words[:, (off // 4).reshape(-1)]
    c = (w >> bit.reshape(-1).astype(np.uint32)) & np.uint32((1 << bits) - 1)
    return c.reshape(n, 32, -1).astype(np.uint8)


def pack_records(kc, ks, kz, vc, vs, vz, d: int, bits: int, G: int) -> np.ndarray:
    """Quantized tokens of one (batch, kv-head) row -> group records.

    kc, vc: codes [T][d] (T a multiple of G); ks, kz: [T/G][d]; vs, vz: [T].
    Returns uint8 [T/G][record_bytes]."""
    T = kc.shape[0]
    ng, ntb = T // G, G // 32
    koff, kbit = key_code_map(d, bits)
    voff, vbit = value_code_map(d, bits)
    cb = tb_code_bytes(d, bits)
    kblk = _pack_tbs(kc.reshape(-1, 32, d), koff, kbit, cb).reshape(ng, ntb * cb)
    vblk = _pack_tbs(vc.reshape(-1, 32, d), voff, vbit, cb).reshape(ng, ntb * cb)
    perm = key_meta_perm(d)
    ksb = np.zeros((ng, d), np.uint16)
    kzb = np.zeros((ng, d), np.uint16)
    ksb[:, perm] = fp16_bits(ks)
    kzb[:, perm] = fp16_bits(kz)
    vperm = value_meta_perm()
    vsb = fp16_bits(vs).reshape(-1, 32).astype(np.uint32)
    vzb = fp16_bits(vz).reshape(-1, 32).astype(np.uint32)
    vmeta = np.zeros((T // 32, 32), np.uint32)
    vmeta[:, vperm] = vsb | (vzb << np.uint32(16))
    vmeta = np.ascontiguousarray(vmeta.reshape(ng, ntb * 32))
    rec = np.concatenate([kblk, vblk, ksb.view(np.uint8), kzb.view(np.uint8),
                          vmeta.view(np.uint8)], axis=1)
    assert rec.shape[1] == record_bytes(d, bits, G)
    return rec


def unpack_records(rec: np.ndarray, d: int, bits: int, G: int):
    """Inverse of pack_records: -> (kc, ks, kz, vc, vs, vz) with fp16 values as
    float64."""
    ng, ntb = rec.shape[0], G // 32
    cb = tb_code_bytes(d, bits)
    koff, kbit = key_code_map(d, bits)
    voff, vbit = value_code_map(d, bits)
    o = 0
    kblk = rec[:, o:o + ntb * cb].reshape(ng * ntb, cb); o += ntb * cb
    vblk = rec[:, o:o + ntb * cb].reshape(ng * ntb, cb); o += ntb * cb
    kc = _unpack_tbs(kblk, koff, kbit, bits).reshape(ng * G, d)
    vc = _unpack_tbs(vblk, voff, vbit, bits).reshape(ng * G, d)
    perm = key_meta_perm(d)
    ks = np.ascontiguousarray(rec[:, o:o + 2 * d]).view(np.float16).astype(np.float64)[:, perm]; o += 2 * d
    kz = np.ascontiguousarray(rec[:, o:o + 2 * d]).view(np.float16).astype(np.float64)[:, perm]; o += 2 * d
    vm = np.ascontiguousarray(rec[:, o:o + 4 * G]).view(np.uint32).reshape(-1, 32)[:, value_meta_perm()]
    vs = (vm & np.uint32(0xFFFF)).astype(np.uint16).view(np.float16).astype(np.float64).reshape(-1)
    vz = (vm >> np.uint32(16)).astype(np.uint16).view(np.float16).astype(np.float64).reshape(-1)
    return kc, ks, kz, vc, vs, vz
