"""libsparsedecode: exact top-k sparse decode attention over a paged GQA bf16 KV cache (sm_100a).

The compute lives in ``libsparsedecode.so`` (hand-written CUDA, C ABI declared in
``include/sparsedecode.h``).  ``binding`` is the thin ctypes layer with the same entry-point
names; ``workloads`` builds seeded synthetic inputs.  Importing the package does not load the
shared library; the first call into ``binding`` does, and raises if the library is missing.
"""
from __future__ import annotations

import importlib

__all__ = ["binding", "workloads"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
