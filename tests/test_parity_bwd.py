"""GPU-vs-oracle parity of the block-sparse attention backward (the gradient of
the attention over a fixed selection) through the C ABI, on bf16 workloads
that span several rows of tiles, ragged tails, every supported G_Q, d and C,
causal and not.

Tolerance: the kernels take the products on bf16 tensor cores. P and dS are
rounded to bf16 (relative 2^-9) before their MMAs, and D = dout.out uses the
forward's bf16 output. Each gradient entry sums many such terms. The bound is
max |gpu - oracle| <= 2e-2 * max |oracle| + 1e-3 per tensor."""
import numpy as np
import pytest
import torch

import _parity as P
import oracle as O
from hierarchical_top_block_mean_b200 import api, workloads

pytestmark = pytest.mark.gpu

BWD_REL = 2e-2
BWD_ABS = 1e-3

_n16 = workloads.PREFILL["needle_16k"]
_c64 = workloads.PREFILL["clustered_64k"]
_tiny = workloads.PREFILL["tiny_noncausal_1k"]

CASES = [
    _n16.with_(name="bwd_G4_needle_1k", N=1100, n_needles=6, seed=6100),
    _c64.with_(name="bwd_G8_ragged", N=1000, H_q=16, H_kv=2, segment=256, seed=6200),
    _c64.with_(name="bwd_d64_C32_K5_G2", N=900, H_q=8, H_kv=4, d=64, C=32, K=5, segment=128, seed=6300),
    _tiny.with_(name="bwd_G1_noncausal", N=700, H_q=2, H_kv=2, d=128, C=64, K=8, dtype="bf16", seed=6400),
    _tiny.with_(name="bwd_G2_B2_causal", B=2, N=555, H_q=4, H_kv=2, d=64, C=32, K=3, causal=True, dtype="bf16",
                seed=6500),
]


def _check(name, got, want):
    err = np.abs(got.astype(np.float64) - want).max()
    bound = BWD_REL * np.abs(want).max() + BWD_ABS
    assert err <= bound, f"{name}: max err {err:.3e} > {bound:.3e}"
    return float(err / max(np.abs(want).max(), 1e-30))


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_attention_backward_parity(w):
    dev = torch.device("cuda")
    x = workloads.prefill_inputs(w, device=dev)
    q, k, v = x["q"], x["k"], x["v"]
    p = api.Prefill(api.Problem.of(q, k, C=w.C, K=w.K, causal=w.causal), dev)
    p(q, k, v)
    g = torch.randn(q.shape, generator=torch.Generator(device=dev).manual_seed(w.seed + 7), device=dev)
    dout = g.to(q.dtype)
    dq, dk, dv = api.sparse_attn_bwd(q, k, v, p.sel, p.out, p.lse, dout, C=w.C, causal=w.causal)
    torch.cuda.synchronize()
    rq, rk, rv = O.attn_bwd(P.ocfg(w), P.host(q), P.host(k), P.host(v), P.host(p.sel).numpy(), P.host(dout))
    rel = {n: _check(f"{w.name} {n}", P.host(a).numpy(), b) for n, a, b in (("dq", dq, rq), ("dk", dk, rk),
                                                                             ("dv", dv, rv))}
    print(w.name, rel)


def test_backward_rejects_fp32_and_small_workspace():
    w = CASES[0]
    dev = torch.device("cuda")
    x = workloads.prefill_inputs(w.with_(dtype="f32"), device=dev)
    q, k, v = x["q"], x["k"], x["v"]
    sel = torch.zeros((w.B, w.H_kv, w.N, w.K), dtype=torch.int32, device=dev)
    lse = torch.zeros((w.B, w.H_q, w.N), dtype=torch.float32, device=dev)
    with pytest.raises(Exception):
        api.sparse_attn_bwd(q, k, v, sel, q, lse, q, C=w.C, causal=w.causal)


@pytest.mark.slow
@pytest.mark.parametrize("name,rows", [("needle_16k", 256), ("needle_256k", 64)])
def test_attention_backward_dq_full_size(name, rows):
    # dk and dv gather every row that selects a block, out of reach of the
    # oracle at full size; dq of a row depends on that row alone, so sampled
    # rows are checked exactly as the small cases are.
    w = workloads.PREFILL[name]
    dev = torch.device("cuda")
    x = workloads.prefill_inputs(w, device=dev)
    q, k, v = x["q"], x["k"], x["v"]
    p = api.Prefill(api.Problem.of(q, k, C=w.C, K=w.K, causal=w.causal), dev)
    p(q, k, v)
    dout = torch.randn(q.shape, generator=torch.Generator(device=dev).manual_seed(w.seed + 7), device=dev).to(q.dtype)
    dq, _, _ = api.sparse_attn_bwd(q, k, v, p.sel, p.out, p.lse, dout, C=w.C, causal=w.causal)
    torch.cuda.synchronize()
    r = P.sample_rows(w, rows)
    ref = O.attn_bwd_dq_rows(P.ocfg(w), P.host(q), P.host(k), P.host(v), r, P.gather_rows(p.sel, r), P.host(dout))
    G = w.H_q // w.H_kv
    d = P.host(dq).numpy()
    hq = r[:, 1:2] * G + np.arange(G)[None, :]
    got = d[r[:, 0:1], hq, r[:, 2:3], :]
    print(name, _check(f"{name} dq", got, ref))
