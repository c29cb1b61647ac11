"""B200-native PISA hot path: mean-pooled key pyramid, coarse-to-fine top-K
block selection, flat single-level selection, block-sparse attention forward
and the decode step, as hand-written sm_100a CUDA behind a C ABI
(include/pisa.h). This package is the thin Python binding over it.

The CUDA library is loaded on first use and its absence is an error: there is
no CPU fallback.
"""
from .api import (DecodeState, Prefill, Problem, build_pyramid, default_scale, launch_count, prefill,
                  pyramid_geometry, pyramid_rows, select, select_flat, sparse_attn_fwd)

__all__ = ["DecodeState", "Prefill", "Problem", "build_pyramid", "default_scale", "launch_count", "prefill",
           "pyramid_geometry", "pyramid_rows", "select", "select_flat", "sparse_attn_fwd"]
