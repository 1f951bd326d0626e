"""B200-native KV-cache compression and compressed-cache decode.

The compute path lives in ``libkvq.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/kvq.h``); ``kvq`` is the thin ctypes binding over it.  Importing the
package does not load the library; ``from kv_cache_quantization_absmax_b200 import kvq``
does, and fails loudly if the library cannot be built or loaded.
"""
import importlib

__all__ = ["kvq", "inputs"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
