"""Lighthouse Attention hot path for NVIDIA B200 (sm_100a).

The compute lives in the shared library ``liblighthouse.so`` (C ABI in
``include/lighthouse.h``); ``lighthouse`` is its thin ctypes binding and
``inputs`` draws the seeded synthetic workloads.  The binding is imported on
first use, so the input generator works without a built library.
"""
from importlib import import_module

__all__ = ["lighthouse", "inputs", "build"]


def __getattr__(name):
    if name in __all__:
        return import_module(f"{__name__}.{name}")
    raise AttributeError(name)
