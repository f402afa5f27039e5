"""ctypes view of libkvq.so (include/kvq.h).  Argument marshalling only."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_CAPACITY, KVQ_ERR_CUDA, KVQ_ERR_DEVICE_STATUS = range(6)
KVQ_KIVI, KVQ_TURBO = 0, 1
KVQ_BF16, KVQ_FP16 = 0, 1
KVQ_DEV_NONFINITE_INPUT, KVQ_DEV_PARAM_OVERFLOW, KVQ_DEV_WAIT_TIMEOUT, KVQ_DEV_BAD_PAGE = 1, 2, 4, 8


class KvqConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "scheme", "bits", "group", "residual", "head_dim", "num_kv_heads", "num_q_heads",
        "batch", "max_seq", "dtype", "qjl_dim", "page_records", "num_pages", "fp8_recent", "anchor_tokens")]


class KvqLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in (
        "total_bytes", "records_offset", "record_bytes", "groups_per_row", "window_offset",
        "ring_tokens", "params_offset", "params_bytes", "status_offset", "pages_per_row", "token_row_bytes",
        "anchor_offset")]


# name -> (restype, argtypes)
_P = ctypes.c_void_p
_SIGS = {
    "kvq_cache_bytes": (ctypes.c_size_t, [ctypes.POINTER(KvqConfig)]),
    "kvq_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(KvqConfig)]),
    "kvq_get_layout": (ctypes.c_int, [ctypes.POINTER(KvqConfig), ctypes.POINTER(KvqLayout)]),
    "kvq_cache_init": (ctypes.c_int, [ctypes.POINTER(KvqConfig), _P, ctypes.c_size_t, _P, ctypes.POINTER(_P)]),
    "kvq_turbo_setup": (ctypes.c_int, [_P, _P, _P, _P]),
    "kvq_turbo_setup_wht": (ctypes.c_int, [_P, _P, _P]),
    "kvq_cache_set_page_table": (ctypes.c_int, [_P, _P]),
    "kvq_quantize_prefill": (ctypes.c_int, [_P, _P, _P, ctypes.c_int32, _P]),
    "kvq_append_token": (ctypes.c_int, [_P, _P, _P, _P]),
    "kvq_decode_attention": (ctypes.c_int, [_P, _P, _P, ctypes.c_float, _P, ctypes.c_size_t, _P]),
    "kvq_decode_attention_static": (ctypes.c_int, [_P, _P, _P, ctypes.c_float, _P]),
    "kvq_append_decode": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_float, _P, ctypes.c_size_t, _P]),
    "kvq_get_status": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_uint32), ctypes.c_int32, _P]),
    "kvq_seq_len": (ctypes.c_int32, [_P]),
    "kvq_quantized_len": (ctypes.c_int32, [_P]),
    "kvq_window_len": (ctypes.c_int32, [_P]),
    "kvq_window_head": (ctypes.c_int32, [_P]),
    "kvq_cache_set_state": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]),
    "kvq_cache_destroy": (None, [_P]),
    "kvq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "kvq_launch_count": (ctypes.c_uint64, []),
    "kvq_debug_set_wait_test": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_int32]),
    "kvq_cuda_error_string": (ctypes.c_char_p, []),
    "kvq_decode_splits": (ctypes.c_int32, [_P]),
    "kvq_decode_partition": (ctypes.c_int32, [_P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _P, ctypes.c_int32, _P]),
}

_lib = None


def load():
    """The loaded library.  Raises when libkvq.so has not been built: there is no
    fallback path."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libkvq.so is not built ({LIB_PATH}); run python -m quantized_kv_cache_18_b200.build")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def exported_symbols():
    return list(_SIGS)


class KvqError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        msg = load().kvq_status_string(code).decode()
        if code == KVQ_ERR_CUDA:
            msg += ": " + load().kvq_cuda_error_string().decode()
        super().__init__(f"{what}: {msg} (status {code})" if what else msg)


def check(code: int, what: str = ""):
    if code != KVQ_OK:
        raise KvqError(code, what)
