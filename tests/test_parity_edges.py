"""Degenerate and boundary shapes through the C ABI, against the oracle: a
single token, fewer tokens than one leaf, one leaf plus one key, K = 1, K at
its maximum of 16 with fewer leaves than K, and a pyramid whose top level is
a lone ragged block. Each runs the pyramid, the pyramid search, the
attention, the exact-score selector and (bf16) the backward."""
import numpy as np
import pytest
import torch

import _parity as P
import oracle as O
from hierarchical_top_block_mean_b200 import api, workloads

pytestmark = pytest.mark.gpu

_base = workloads.PREFILL["needle_16k"].with_(n_needles=0, structure="iid")

EDGES = [
    _base.with_(name="one_token", N=1, seed=8100),
    _base.with_(name="under_one_leaf", N=37, seed=8200),
    _base.with_(name="one_leaf_plus_one", N=65, seed=8300),
    _base.with_(name="K1", N=1000, K=1, seed=8400),
    _base.with_(name="K16_few_leaves", N=700, K=16, seed=8500),   # 11 leaves < K
    _base.with_(name="ragged_top", N=64 * 33 + 5, K=4, seed=8600),  # 34 leaves: lone top-level blocks
    _base.with_(name="f32_one_leaf_plus_one", N=33, C=32, d=64, H_q=4, H_kv=2, K=2, dtype="f32", seed=8700),
    _base.with_(name="noncausal_K1_G8", N=300, H_q=16, H_kv=2, K=1, causal=False, seed=8800),
]


@pytest.mark.parametrize("w", EDGES, ids=lambda w: w.name)
def test_edge_shapes(w):
    dev = torch.device("cuda")
    x = workloads.prefill_inputs(w, device=dev)
    q, k, v = x["q"], x["k"], x["v"]
    p = api.Prefill(api.Problem.of(q, k, C=w.C, K=w.K, causal=w.causal), dev)
    p(q, k, v)
    xsel = api.select_exact(q, k, C=w.C, K=w.K, causal=w.causal)
    torch.cuda.synchronize()
    qh, kh, vh = P.host(q), P.host(k), P.host(v)
    pyr_ref = P.check_pyramid(w, kh, P.host(p.pyr))
    rows = P.sample_rows(w, None)
    cfg = P.ocfg(w)
    sel_ref, gap = O.select_rows(cfg, qh, kh, pyr_ref, rows)
    sel_gpu = P.gather_rows(p.sel, rows)
    n, n_ex, bad, _ = P.compare_selection(w, sel_gpu, sel_ref, gap)
    assert bad == 0, f"{w.name}: {bad} selection mismatches of {n}"
    ex_ref, ex_gap = O.select_exact_rows(cfg, qh, kh, rows)
    _, _, xbad, _ = P.compare_selection(w, P.gather_rows(xsel, rows), ex_ref, ex_gap)
    assert xbad == 0, f"{w.name}: exact selector {xbad} mismatches"
    out_ref, lse_ref = O.attn_rows(cfg, qh, kh, vh, rows, sel_gpu)
    P.check_attention(w, P.gather_out(w, p.out, rows), P.gather_lse(w, p.lse, rows), out_ref, lse_ref)
    if w.dtype == "bf16":
        dout = torch.randn(q.shape, generator=torch.Generator(device=dev).manual_seed(w.seed + 1),
                           device=dev).to(q.dtype)
        dq, dk, dv = api.sparse_attn_bwd(q, k, v, p.sel, p.out, p.lse, dout, C=w.C, causal=w.causal)
        torch.cuda.synchronize()
        rq, rk, rv = O.attn_bwd(cfg, qh, kh, vh, P.host(p.sel).numpy(), P.host(dout))
        for name, got, want in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            err = np.abs(P.host(got).numpy() - want).max()
            assert err <= 2e-2 * np.abs(want).max() + 1e-3, f"{w.name} {name}: {err:.3e}"
