"""NOSA sparse decode attention for NVIDIA B200 (sm_100a).

The compute path is the CUDA library ``libnosa_b200.so`` (built from
``csrc/``); :mod:`long_context_decode_nosa_b200.nosa` is its thin ctypes
binding.  Nothing here computes on the CPU: every call fails loudly when the
library or a CUDA device is missing.
"""
from __future__ import annotations

import importlib

__all__ = ["nosa", "inputs"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
