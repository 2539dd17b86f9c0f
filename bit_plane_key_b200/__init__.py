"""Fathom on B200: per-query variable-depth key scan over a bit-plane 4-bit K cache.

The compute path is libfathom.so (hand-written CUDA for sm_100a behind the C ABI
in include/fathom.h); `bit_plane_key_b200.fathom` is its Python binding.  The
binding is imported on first use, and importing it without the built library
raises ImportError: there is no fallback path.
"""
import importlib

__all__ = ["fathom", "build"]


def __getattr__(name):
    if name in ("fathom", "build"):
        return importlib.import_module("." + name, __name__)
    mod = importlib.import_module(".fathom", __name__)
    return getattr(mod, name)
