"""Fine-grained FP8 (E4M3) quantisation and block-scaled FP8 GEMM for B200 (sm_100a).

The compute lives in ``libfp8q.so`` (hand-written CUDA behind a C ABI declared in
``include/fp8q.h``); :mod:`.ops` is the thin ctypes binding.  Importing the package does not
load the library; the first use of an op does, and raises if it is missing.
"""
import importlib

__all__ = ["ops", "synth"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
