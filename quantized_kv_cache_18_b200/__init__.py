"""Quantized KV cache with decode attention read straight from the packed cache,
for NVIDIA B200 (sm_100a).

The compute lives in libkvq.so (C ABI in include/kvq.h); `QuantizedKVCache`
wraps it for PyTorch callers.  Importing this package does not load the
library; the first cache construction does, and fails loudly if it was not
built.
"""
from . import workloads  # noqa: F401  (pure numpy, no library load)

__all__ = ["QuantizedKVCache", "workloads"]


def __getattr__(name):
    if name in ("QuantizedKVCache", "make_config", "config_from_workload", "cache_bytes", "workspace_bytes",
                "layout", "launch_count"):
        from . import cache
        return getattr(cache, name)
    raise AttributeError(name)
