"""B200-native PISA hot path: mean-pooled key pyramid, coarse-to-fine top-K
block selection, flat and exact-score single-level selection, block-sparse
attention forward and backward, the decode step (dense or paged caches) and
sequence-parallel prefill over query shards, as hand-written sm_100a CUDA
behind a C ABI (include/pisa.h). This package is the thin Python binding over
it.

The CUDA library is loaded on first use and its absence is an error: there is
no CPU fallback.
"""
from .api import (DecodeState, PagedDecodeState, Prefill, PrefillShard, PrefillStream, Problem, build_pyramid, default_scale, launch_count,
                  prefill, pyramid_geometry, pyramid_rows, select, select_exact, select_flat, select_span,
                  sparse_attn_bwd, sparse_attn_fwd, sparse_attn_fwd_span)
from .seqpar import SeqParallelPrefill, gather_sequence, shard_span

__all__ = ["DecodeState", "PagedDecodeState", "Prefill", "PrefillShard", "PrefillStream", "Problem", "SeqParallelPrefill", "build_pyramid",
           "default_scale", "gather_sequence", "launch_count", "prefill", "pyramid_geometry", "pyramid_rows", "select",
           "select_exact", "select_flat", "select_span", "shard_span", "sparse_attn_bwd", "sparse_attn_fwd",
           "sparse_attn_fwd_span"]
