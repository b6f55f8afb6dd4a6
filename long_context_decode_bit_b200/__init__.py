"""Fathom top-k key scan for sparse long-context decoding, on B200 (sm_100a).

The compute path lives in ``libfathom.so`` (hand-written CUDA behind a C
ABI, declared in ``include/fathom.h``); :mod:`.fathom` is its thin ctypes
binding.  :mod:`.inputs` draws seeded synthetic workloads and
:mod:`.accounting` holds the byte-accounting model used by the benchmark.
"""
__all__ = ["fathom", "inputs", "accounting"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
