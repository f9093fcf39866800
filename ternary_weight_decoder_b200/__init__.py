"""B200-native ternary-weight linear layer (1.58-bit decoder projections).

The compute path lives in ``libternary_decoder.so`` (CUDA for sm_100a behind a
C ABI declared in ``include/ternary_decoder.h``); ``api`` is the thin Python
binding over it and raises ImportError when the library is missing.
"""
import importlib

__all__ = ["api", "synth"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
