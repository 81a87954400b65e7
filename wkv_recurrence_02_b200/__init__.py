"""B200-native WKV recurrences (RWKV-4 and Eagle/Finch WKV-6) behind a C ABI.

The compute lives in ``libwkv.so`` (hand-written CUDA for sm_100a, built by
``wkv_recurrence_02_b200.build``); ``wkv_recurrence_02_b200.ops`` is the thin
ctypes binding.  Importing this package does not load the library; calling an
op does, and fails loudly if it is missing or no CUDA device is present.
"""

__all__ = ["ops", "inputs"]


def __getattr__(name):
    if name in ("ops", "inputs", "build"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
