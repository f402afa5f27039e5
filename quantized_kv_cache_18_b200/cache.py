"""Python face of the library: a quantized KV cache over caller-owned device
memory.  Every step runs in libkvq.so's kernels; this module only allocates
device buffers with PyTorch, picks the current stream and marshals pointers."""
from __future__ import annotations

import ctypes
import math
from typing import Optional

import torch

from . import _lib as L


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def make_config(scheme: str, bits: int, group: int, residual: int, head_dim: int, num_kv_heads: int,
                num_q_heads: int, batch: int, max_seq: int, dtype: str, qjl_dim: int = 0,
                page_records: int = 0, num_pages: int = 0, fp8_recent: int = 0,
                anchor_tokens: int = 0) -> L.KvqConfig:
    return L.KvqConfig(L.KVQ_KIVI if scheme == "kivi" else L.KVQ_TURBO, bits, group, residual, head_dim,
                       num_kv_heads, num_q_heads, batch, max_seq,
                       L.KVQ_BF16 if dtype == "bf16" else L.KVQ_FP16, qjl_dim, page_records, num_pages,
                       fp8_recent, anchor_tokens)


def config_from_workload(w, max_seq: Optional[int] = None, page_records: int = 0,
                         num_pages: int = 0) -> L.KvqConfig:
    return make_config(w.scheme, w.bits, w.group, w.residual, w.head_dim, w.num_kv_heads, w.num_q_heads,
                       w.batch, max_seq if max_seq is not None else w.max_seq, w.dtype,
                       w.qjl_dim if w.scheme == "turbo" else 0, page_records, num_pages,
                       1 if w.fp8_recent else 0, w.anchor_tokens)


def cache_bytes(cfg: L.KvqConfig) -> int:
    return int(L.load().kvq_cache_bytes(ctypes.byref(cfg)))


def workspace_bytes(cfg: L.KvqConfig) -> int:
    return int(L.load().kvq_workspace_bytes(ctypes.byref(cfg)))


def decode_partition(cfg: L.KvqConfig, n_groups: int, r: int, sms: int):
    """The decode launch's work partition (kvq_decode_partition): the first
    global item of each CTA followed by the end, and the items per row.
    Host only."""
    buf = (ctypes.c_int32 * 161)()
    n_items = ctypes.c_int32()
    n = L.load().kvq_decode_partition(ctypes.byref(cfg), n_groups, r, sms, buf, 161, ctypes.byref(n_items))
    if n <= 0:
        raise ValueError("kvq_decode_partition: unsupported arguments")
    return list(buf[:n + 1]), int(n_items.value)


def layout(cfg: L.KvqConfig) -> L.KvqLayout:
    out = L.KvqLayout()
    L.check(L.load().kvq_get_layout(ctypes.byref(cfg), ctypes.byref(out)), "kvq_get_layout")
    return out


class QuantizedKVCache:
    """One layer's quantized KV cache for a batch of equal-length sequences."""

    def __init__(self, cfg: L.KvqConfig, device: str = "cuda", buffer: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None):
        self.lib = L.load()
        self.cfg = cfg
        self.nbytes = cache_bytes(cfg)
        if self.nbytes == 0:
            raise L.KvqError(L.KVQ_ERR_UNSUPPORTED, "kvq_cache_bytes")
        self.layout = layout(cfg)
        self.buf = buffer if buffer is not None else torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        wsb = workspace_bytes(cfg)
        self.ws = workspace if workspace is not None else torch.empty(max(wsb, 16), dtype=torch.uint8,
                                                                       device=self.buf.device)
        self.handle = ctypes.c_void_p()
        L.check(self.lib.kvq_cache_init(ctypes.byref(cfg), _ptr(self.buf), self.nbytes, _stream_ptr(stream),
                                        ctypes.byref(self.handle)), "kvq_cache_init")

    # ------------------------------------------------------------------ lifecycle
    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            self.lib.kvq_cache_destroy(self.handle)
            self.handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------------ state
    @property
    def seq_len(self) -> int:
        return int(self.lib.kvq_seq_len(self.handle))

    @property
    def quantized_len(self) -> int:
        return int(self.lib.kvq_quantized_len(self.handle))

    @property
    def window_len(self) -> int:
        return int(self.lib.kvq_window_len(self.handle))

    @property
    def window_head(self) -> int:
        return int(self.lib.kvq_window_head(self.handle))

    @property
    def decode_splits(self) -> int:
        return int(self.lib.kvq_decode_splits(self.handle))

    def set_state(self, seq_len: int, quantized_len: int, window_head: int):
        L.check(self.lib.kvq_cache_set_state(self.handle, seq_len, quantized_len, window_head), "kvq_cache_set_state")

    def turbo_setup(self, rot_gauss: torch.Tensor, qjl_gauss: torch.Tensor, stream=None):
        """TurboQuant scheme: derive the rotation, codebook and sketch tables on
        the device from two float32 N(0, 1) draws, [d][d] and [m][d]."""
        c = self.cfg
        for t, shape, what in ((rot_gauss, (c.head_dim, c.head_dim), "rot_gauss"),
                               (qjl_gauss, (c.qjl_dim, c.head_dim), "qjl_gauss")):
            if t.device != self.buf.device or t.dtype != torch.float32 or not t.is_contiguous():
                raise ValueError(f"{what}: needs a contiguous float32 tensor on {self.buf.device}")
            if tuple(t.shape) != shape:
                raise ValueError(f"{what}: shape {tuple(t.shape)} != {shape}")
        L.check(self.lib.kvq_turbo_setup(self.handle, _ptr(rot_gauss), _ptr(qjl_gauss), _stream_ptr(stream)),
                "kvq_turbo_setup")

    def set_page_table(self, table: torch.Tensor):
        """Paged caches: the block table, int32 [B*Hkv][pages_per_row] on the
        cache's device (kept referenced by this object)."""
        c, lay = self.cfg, self.layout
        shape = (c.batch * c.num_kv_heads, lay.pages_per_row)
        if table.device != self.buf.device or table.dtype != torch.int32 or not table.is_contiguous():
            raise ValueError(f"page table: needs a contiguous int32 tensor on {self.buf.device}")
        if tuple(table.shape) != shape:
            raise ValueError(f"page table: shape {tuple(table.shape)} != {shape}")
        L.check(self.lib.kvq_cache_set_page_table(self.handle, _ptr(table)), "kvq_cache_set_page_table")
        self.page_table = table

    def row_records(self, row: int, n: int) -> torch.Tensor:
        """[n][record_bytes] uint8 copy of a row's first n records, through the
        block table for a paged cache."""
        c, lay = self.cfg, self.layout
        if c.page_records == 0:
            return self.records_view()[row, :n]
        pool = self.buf[lay.records_offset:lay.records_offset + c.num_pages * c.page_records * lay.record_bytes]
        pool = pool.view(c.num_pages * c.page_records, lay.record_bytes)
        k = torch.arange(n, device=self.buf.device)
        pages = self.page_table[row].long()[k // c.page_records]
        return pool[pages * c.page_records + k % c.page_records]

    def turbo_setup_wht(self, qjl_gauss: torch.Tensor, stream=None):
        """TurboQuant scheme with the Walsh-Hadamard rotation H / sqrt(d): the
        codebook and sketch tables from the [m][d] float32 N(0, 1) draw."""
        c = self.cfg
        if qjl_gauss.device != self.buf.device or qjl_gauss.dtype != torch.float32 or not qjl_gauss.is_contiguous():
            raise ValueError(f"qjl_gauss: needs a contiguous float32 tensor on {self.buf.device}")
        if tuple(qjl_gauss.shape) != (c.qjl_dim, c.head_dim):
            raise ValueError(f"qjl_gauss: shape {tuple(qjl_gauss.shape)} != {(c.qjl_dim, c.head_dim)}")
        L.check(self.lib.kvq_turbo_setup_wht(self.handle, _ptr(qjl_gauss), _stream_ptr(stream)),
                "kvq_turbo_setup_wht")

    # ------------------------------------------------------------------ the three calls
    def _check_16(self, t: torch.Tensor, shape, what: str):
        if t.device != self.buf.device or not t.is_contiguous() or t.element_size() != 2:
            raise ValueError(f"{what}: needs a contiguous 16-bit tensor on {self.buf.device}")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{what}: shape {tuple(t.shape)} != {tuple(shape)}")

    def prefill(self, k: torch.Tensor, v: torch.Tensor, stream=None):
        c = self.cfg
        S = k.shape[2]
        shape = (c.batch, c.num_kv_heads, S, c.head_dim)
        self._check_16(k, shape, "k")
        self._check_16(v, shape, "v")
        L.check(self.lib.kvq_quantize_prefill(self.handle, _ptr(k), _ptr(v), S, _stream_ptr(stream)),
                "kvq_quantize_prefill")

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None):
        c = self.cfg
        shape = (c.batch, c.num_kv_heads, c.head_dim)
        self._check_16(k_new, shape, "k_new")
        self._check_16(v_new, shape, "v_new")
        L.check(self.lib.kvq_append_token(self.handle, _ptr(k_new), _ptr(v_new), _stream_ptr(stream)),
                "kvq_append_token")

    def attention(self, q: torch.Tensor, out: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                  stream=None) -> torch.Tensor:
        c = self.cfg
        self._check_16(q, (c.batch, c.num_q_heads, c.head_dim), "q")
        if out is None:
            out = torch.empty((c.batch, c.num_q_heads, c.head_dim), dtype=torch.float32, device=self.buf.device)
        if scale is None:
            scale = 1.0 / math.sqrt(c.head_dim)
        L.check(self.lib.kvq_decode_attention(self.handle, _ptr(q), _ptr(out), float(scale), _ptr(self.ws),
                                              self.ws.numel(), _stream_ptr(stream)), "kvq_decode_attention")
        return out

    def append_attention(self, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor,
                         out: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                         stream=None) -> torch.Tensor:
        """append(k_new, v_new) then attention(q) as one decode step
        (kvq_append_decode: one kernel launch unless the step flushes)."""
        c = self.cfg
        shape = (c.batch, c.num_kv_heads, c.head_dim)
        self._check_16(k_new, shape, "k_new")
        self._check_16(v_new, shape, "v_new")
        self._check_16(q, (c.batch, c.num_q_heads, c.head_dim), "q")
        if out is None:
            out = torch.empty((c.batch, c.num_q_heads, c.head_dim), dtype=torch.float32, device=self.buf.device)
        if scale is None:
            scale = 1.0 / math.sqrt(c.head_dim)
        L.check(self.lib.kvq_append_decode(self.handle, _ptr(k_new), _ptr(v_new), _ptr(q), _ptr(out), float(scale),
                                           _ptr(self.ws), self.ws.numel(), _stream_ptr(stream)),
                "kvq_append_decode")
        return out

    def status(self, clear: bool = False, stream=None) -> int:
        bits = ctypes.c_uint32(0)
        self.lib.kvq_get_status(self.handle, ctypes.byref(bits), 1 if clear else 0, _stream_ptr(stream))
        return int(bits.value)

    # ------------------------------------------------------------------ raw views (tests, checkpoints)
    def records_view(self) -> torch.Tensor:
        """[B*Hkv][groups_per_row][record_bytes] uint8 view of the packed groups."""
        c, lay = self.cfg, self.layout
        n = c.batch * c.num_kv_heads * lay.groups_per_row * lay.record_bytes
        return self.buf[lay.records_offset:lay.records_offset + n].view(
            c.batch * c.num_kv_heads, lay.groups_per_row, lay.record_bytes)

    def params_view(self) -> torch.Tensor:
        """uint8 view of the TurboQuant parameter block (empty for KIVI)."""
        lay = self.layout
        return self.buf[lay.params_offset:lay.params_offset + lay.params_bytes]

    def fp8_ring_view(self) -> torch.Tensor:
        """fp8_recent caches: [B*Hkv][2][ring_tokens][144] uint8 FP8 token rows of the window."""
        c, lay = self.cfg, self.layout
        n = c.batch * c.num_kv_heads * 2 * lay.ring_tokens * lay.token_row_bytes
        return self.buf[lay.window_offset:lay.window_offset + n].view(
            c.batch * c.num_kv_heads, 2, lay.ring_tokens, lay.token_row_bytes)

    def anchor_view(self) -> torch.Tensor:
        """fp8_recent caches: [B*Hkv][2][A][144] uint8 FP8 token rows of the anchors."""
        c, lay = self.cfg, self.layout
        n = c.batch * c.num_kv_heads * 2 * c.anchor_tokens * lay.token_row_bytes
        return self.buf[lay.anchor_offset:lay.anchor_offset + n].view(
            c.batch * c.num_kv_heads, 2, c.anchor_tokens, lay.token_row_bytes)

    def ring_view(self) -> torch.Tensor:
        """[B*Hkv][2][ring_tokens][d] 16-bit patterns (as int16) of the residual rings."""
        c, lay = self.cfg, self.layout
        n = c.batch * c.num_kv_heads * 2 * lay.ring_tokens * c.head_dim * 2
        return self.buf[lay.window_offset:lay.window_offset + n].view(torch.int16).view(
            c.batch * c.num_kv_heads, 2, lay.ring_tokens, c.head_dim)


def launch_count() -> int:
    return int(L.load().kvq_launch_count())


def turbo_setup_from_workload(cache: "QuantizedKVCache", w, stream=None):
    """TurboQuant set-up of a cache with the workload's seeded draws: the QR
    rotation from the [d][d] draw, or the Walsh-Hadamard one (w.rotation)."""
    from . import workloads as W
    dev = cache.buf.device
    qjl = torch.from_numpy(W.gaussian_matrix(w, "qjl", w.qjl_dim, w.head_dim)).to(dev)
    if w.rotation == "wht":
        cache.turbo_setup_wht(qjl, stream)
    else:
        rot = torch.from_numpy(W.gaussian_matrix(w, "rot", w.head_dim, w.head_dim)).to(dev)
        cache.turbo_setup(rot, qjl, stream)
