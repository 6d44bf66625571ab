"""B200-native MicroAdam optimizer step (sm_100a CUDA kernels behind a C ABI).

The method is the one on "MicroAdam (Sparse-Gradient Adaptive Optimization
with Quantized Error Feedback)": a 4-bit error-feedback buffer, a per-block
Top-k of gradient + error, a circular window of m sparse gradients (int16
indices, bf16 values) and Adam statistics recomputed from that window.

Every step of the path runs in ``libmua.so`` (built in-tree by
``compressed_state_optimizer_b200/build.py``); this package only marshals
arguments through ctypes. Importing it fails loudly if the library is absent:
there is no CPU fallback.
"""
from __future__ import annotations

from .binding import (MUA_STATUS_NONFINITE, MicroAdam, MuaError, Layout, library,
                      library_path, strerror)

__all__ = ["MicroAdam", "MuaError", "Layout", "library", "library_path", "strerror",
           "MUA_STATUS_NONFINITE"]
