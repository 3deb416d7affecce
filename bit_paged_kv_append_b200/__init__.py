"""B200-native SAW-INT4 paged KV cache: fused BDR + token-wise INT4 append and paged GQA decode.

The compute lives in ``libkvq.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/kvq.h``); ``bit_paged_kv_append_b200.kvq`` is the thin ctypes
binding with the same entry-point names.  Importing this package does not load the
library; the first call into ``kvq`` does, and raises if it is missing.
"""

__all__ = ["kvq", "synth"]


def __getattr__(name):
    if name in ("kvq", "synth"):
        import importlib

        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
