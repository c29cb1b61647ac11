"""pisa_select_noalloc: the allocation-free selection entry point.

It exists for callers that cannot allocate device memory when they select
(for example a plugin that its host framework hands only input and output
buffers, or a service whose memory pool owns the whole GPU). It must select
exactly what pisa_select selects with a caller workspace, on consecutive
calls that share its library-owned scratch array. This file is collected last
so that a run stopping at the first failure has run every other test.
"""
import ctypes

import pytest
import torch

from hierarchical_top_block_mean_b200 import _lib, api, workloads


def _inputs(seed, **kw):
    base = dict(name=f"noalloc_{seed}", N=3000, n_needles=8, seed=seed)
    base.update(kw)
    w = workloads.PREFILL["needle_16k"].with_(**base)
    x = workloads.prefill_inputs(w, device=torch.device("cuda"))
    return w, x


def _noalloc(w, x, pyr):
    pr = api.Problem.of(x["q"], x["k"], C=w.C, K=w.K, causal=w.causal)
    sel = torch.full((w.B, w.H_kv, w.N, w.K), -7, dtype=torch.int32, device="cuda")
    score = torch.full(sel.shape, -7.0, dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = _lib.lib().pisa_select_noalloc(ctypes.byref(pr.cstruct()), ctypes.c_void_p(x["q"].data_ptr()),
                                        ctypes.c_void_p(x["k"].data_ptr()), ctypes.c_void_p(pyr.data_ptr()),
                                        ctypes.c_void_p(sel.data_ptr()), ctypes.c_void_p(score.data_ptr()), stream)
    assert st == 0, _lib.STATUS_NAMES.get(st, st)
    return sel, score


def _with_workspace(w, x, pyr):
    score = torch.empty((w.B, w.H_kv, w.N, w.K), dtype=torch.float32, device="cuda")
    sel = api.select(x["q"], x["k"], pyr, C=w.C, K=w.K, causal=w.causal, score=score)
    return sel, score


@pytest.mark.gpu
def test_noalloc_matches_workspace_select_on_two_calls():
    # Two calls in a row, different inputs, one shared scratch array. The
    # first has G_Q = 4 (mma.sync leaf scorer); the second G_Q = 8 with
    # d = 128, C = 64, which takes the tcgen05 leaf scorer and its work lists.
    for seed, kw in ((6101, {}), (6102, dict(H_q=16, H_kv=2, N=3100))):
        w, x = _inputs(seed, **kw)
        pyr = api.build_pyramid(x["k"], C=w.C)
        want_sel, want_score = _with_workspace(w, x, pyr)
        got_sel, got_score = _noalloc(w, x, pyr)
        torch.cuda.synchronize()
        assert torch.equal(got_sel, want_sel)  # block indices: bit-exact
        assert torch.allclose(got_score, want_score, rtol=0, atol=1e-6, equal_nan=True)


def test_noalloc_rejects_oversized_and_fp32_before_launch():
    lib = _lib.lib()
    dummy = ctypes.c_void_p(256)
    before = lib.pisa_launch_count()
    big = _lib.Config(1, 262144, 16, 2, 128, 64, 2, 16, 4, 1, _lib.DTYPE_BF16, 0.0)
    assert lib.pisa_select_workspace_bytes(ctypes.byref(big)) > (64 << 20)
    assert lib.pisa_select_noalloc(ctypes.byref(big), dummy, dummy, dummy, dummy, None, None) == 3
    f32 = _lib.Config(1, 1024, 4, 1, 64, 32, 2, 4, 4, 0, _lib.DTYPE_F32, 0.0)
    assert lib.pisa_select_noalloc(ctypes.byref(f32), dummy, dummy, dummy, dummy, None, None) == 2
    assert lib.pisa_launch_count() == before
