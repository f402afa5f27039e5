"""The C-ABI library loads, exports every symbol include/kvq.h declares, and its
host-only paths (sizes, layout, argument validation) behave as documented.
No GPU: nothing here launches a kernel."""
import ctypes
import os
import re

import pytest

from quantized_kv_cache_18_b200 import _lib as L
from quantized_kv_cache_18_b200 import build as kbuild
from quantized_kv_cache_18_b200.cache import config_from_workload, make_config
from quantized_kv_cache_18_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return L.load()


def _header_functions():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = _header_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(names) == sorted(L.exported_symbols())


def test_symbols_with_nm(lib):
    out = os.popen(f"nm -D --defined-only {L.LIB_PATH}").read()
    for n in _header_functions():
        assert re.search(rf"\bT {n}\b", out), n


def test_cache_bytes_match_layout(lib):
    for name, w in WORKLOADS.items():
        if w.scheme != "kivi":
            continue
        cfg = config_from_workload(w)
        n = lib.kvq_cache_bytes(ctypes.byref(cfg))
        lay = L.KvqLayout()
        assert lib.kvq_get_layout(ctypes.byref(cfg), ctypes.byref(lay)) == L.KVQ_OK
        rows = w.batch * w.num_kv_heads
        rec = w.group * w.head_dim * w.bits // 4 + 4 * w.head_dim + 4 * w.group
        assert lay.record_bytes == rec
        assert lay.groups_per_row == (w.max_seq - w.residual) // w.group
        assert lay.ring_tokens == w.residual + w.group
        assert lay.window_offset >= rows * lay.groups_per_row * rec
        assert lay.status_offset >= lay.window_offset + rows * 2 * lay.ring_tokens * w.head_dim * 2
        assert n == lay.total_bytes and n % 256 == 0
        assert lib.kvq_workspace_bytes(ctypes.byref(cfg)) > 0


@pytest.mark.parametrize("field,value", [
    ("bits", 3), ("group", 48), ("head_dim", 96), ("residual", 40), ("num_q_heads", 12),
    ("batch", 0), ("max_seq", 0), ("dtype", 7), ("scheme", 9)])
def test_unsupported_configs_are_rejected(lib, field, value):
    cfg = make_config("kivi", 2, 32, 32, 64, 2, 4, 1, 512, "fp16")
    setattr(cfg, field, value)
    assert lib.kvq_cache_bytes(ctypes.byref(cfg)) == 0
    assert lib.kvq_workspace_bytes(ctypes.byref(cfg)) == 0
    lay = L.KvqLayout()
    assert lib.kvq_get_layout(ctypes.byref(cfg), ctypes.byref(lay)) == L.KVQ_ERR_UNSUPPORTED
    h = ctypes.c_void_p()
    assert lib.kvq_cache_init(ctypes.byref(cfg), ctypes.c_void_p(256), 1 << 30, None,
                              ctypes.byref(h)) == L.KVQ_ERR_UNSUPPORTED


def test_null_and_misaligned_arguments_return_before_any_launch(lib):
    cfg = make_config("kivi", 2, 32, 32, 64, 2, 4, 1, 512, "fp16")
    h = ctypes.c_void_p()
    n = lib.kvq_cache_bytes(ctypes.byref(cfg))
    assert lib.kvq_cache_init(None, ctypes.c_void_p(256), n, None, ctypes.byref(h)) == L.KVQ_ERR_INVALID_ARG
    assert lib.kvq_cache_init(ctypes.byref(cfg), None, n, None, ctypes.byref(h)) == L.KVQ_ERR_INVALID_ARG
    assert lib.kvq_cache_init(ctypes.byref(cfg), ctypes.c_void_p(256 + 16), n, None,
                              ctypes.byref(h)) == L.KVQ_ERR_INVALID_ARG          # not 256-aligned
    assert lib.kvq_cache_init(ctypes.byref(cfg), ctypes.c_void_p(256), n - 1, None,
                              ctypes.byref(h)) == L.KVQ_ERR_INVALID_ARG          # too small
    assert lib.kvq_quantize_prefill(None, ctypes.c_void_p(16), ctypes.c_void_p(16), 4, None) == L.KVQ_ERR_INVALID_ARG
    assert lib.kvq_append_token(None, ctypes.c_void_p(16), ctypes.c_void_p(16), None) == L.KVQ_ERR_INVALID_ARG
    assert lib.kvq_decode_attention(None, ctypes.c_void_p(16), ctypes.c_void_p(16), 0.125, ctypes.c_void_p(16),
                                    1 << 20, None) == L.KVQ_ERR_INVALID_ARG
    assert lib.kvq_get_status(None, None, 0, None) == L.KVQ_ERR_INVALID_ARG
    assert lib.kvq_cache_set_state(None, 1, 0, 0) == L.KVQ_ERR_INVALID_ARG
    assert lib.kvq_seq_len(None) == -1 and lib.kvq_decode_splits(None) == -1
    lib.kvq_cache_destroy(None)


def test_status_strings(lib):
    for code in range(6):
        assert lib.kvq_status_string(code).decode()
    assert lib.kvq_status_string(99).decode() == "unknown status"


def test_launch_counter_starts_without_device_work(lib):
    assert lib.kvq_launch_count() >= 0


def test_turbo_layout(lib):
    """TurboQuant-style cache: 4032-byte token blocks (3-bit codes of keys and
    values, 128 sketch bits, fp16 norms and gammas), a parameter block for the
    rotation, its transpose, the sketch and the codebook."""
    w = WORKLOADS["tq"]
    cfg = config_from_workload(w)
    lay = L.KvqLayout()
    assert lib.kvq_get_layout(ctypes.byref(cfg), ctypes.byref(lay)) == L.KVQ_OK
    rows = w.batch * w.num_kv_heads
    assert lay.record_bytes == 4032 == 2 * 1664 + 512 + 128 + 64
    assert lay.groups_per_row == (w.max_seq - w.residual) // 32
    # Pi, Pi^T, S^T, tables, (S Pi)^T, then the fp16 and the bf16 sets of four tensor-core operand images
    assert lay.params_bytes == 4 * 128 * 128 * 4 + 128 + 256 + 2 * 4 * 128 * 128 * 2
    assert lay.params_offset % 256 == 0 and lay.params_offset >= lay.window_offset + rows * 2 * lay.ring_tokens * 256
    assert lay.status_offset >= lay.params_offset + lay.params_bytes
    assert lib.kvq_cache_bytes(ctypes.byref(cfg)) == lay.total_bytes
    # rotated query fragments (8 KiB per row) + (2 rows + SMs) partial slots
    ws = lib.kvq_workspace_bytes(ctypes.byref(cfg))
    g = w.gqa
    assert ws >= rows * 8192 + 2 * rows * g * 130 * 4


@pytest.mark.parametrize("field,value", [("bits", 2), ("group", 64), ("head_dim", 64), ("qjl_dim", 64)])
def test_unsupported_turbo_configs_are_rejected(lib, field, value):
    cfg = config_from_workload(WORKLOADS["tq"])
    setattr(cfg, field, value)
    assert lib.kvq_cache_bytes(ctypes.byref(cfg)) == 0


def test_missing_library_fails_loudly(monkeypatch):
    """No fallback: without libkvq.so every call path raises."""
    from quantized_kv_cache_18_b200 import _lib as L
    monkeypatch.setattr(L, "_lib", None)
    monkeypatch.setattr(L, "LIB_PATH", os.path.join(ROOT, "no_such_dir", "libkvq.so"))
    with pytest.raises(RuntimeError, match="not built"):
        L.load()
