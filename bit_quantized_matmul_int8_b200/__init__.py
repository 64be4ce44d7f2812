"""LLM.int8() mixed-precision linear layer for NVIDIA B200 (sm_100a).

The compute lives in ``libint8lt.so`` (CUDA, built in-tree by ``build.py``);
``_lib`` is its ctypes binding. ``workloads`` draws the seeded synthetic inputs.
"""
from __future__ import annotations

__all__ = ["Int8Linear", "int8lt_prepare_weight", "int8lt_quantize_rows", "int8lt_forward",
           "int8lt_workspace_size", "workspace", "int8lt_quantize_rows_zp",
           "int8lt_prepare_weight_zp", "int8lt_forward_zp"]


def __getattr__(name):  # import torch and the library only when used
    if name in __all__:
        from . import _lib
        return getattr(_lib, name)
    raise AttributeError(name)
