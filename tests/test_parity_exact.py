"""GPU-vs-oracle parity of the exact-score flat selector (every usable leaf
scored by its raw-key LSE summed over the group, then top K) through the C ABI,
on both kernels: the tcgen05 tile kernel (bf16, d = 128, C = 64, any G_Q) and
the warp-per-row kernel (every other configuration). Also reports how many of
the exact top-K leaves the pyramid search keeps (recall), which is a property
of the method, not a parity condition."""
import numpy as np
import pytest
import torch

import _parity as P
import oracle as O
from hierarchical_top_block_mean_b200 import api, workloads

pytestmark = pytest.mark.gpu

_n16 = workloads.PREFILL["needle_16k"]
_c64 = workloads.PREFILL["clustered_64k"]
_tiny = workloads.PREFILL["tiny_noncausal_1k"]

SMALL = [
    # tcgen05 kernel: G_Q = 4, 8, 1, 2; causal and not; ragged tails.
    _n16.with_(name="umma_G4_needle_3k", N=3000, n_needles=12, seed=4100),
    _c64.with_(name="umma_G8_4k", N=4160, H_q=16, H_kv=2, segment=512, seed=4200),
    _tiny.with_(name="umma_G1_noncausal", N=1500, H_q=2, H_kv=2, d=128, C=64, K=8, dtype="bf16", seed=4300),
    _tiny.with_(name="umma_G2_K3_ragged", N=1101, H_q=4, H_kv=2, d=128, C=64, K=3, causal=True, dtype="bf16",
                seed=4400),
    _n16.with_(name="umma_G4_short", N=700, K=16, n_needles=2, seed=4500),  # fewer leaves than K early on
    # warp-per-row kernel.
    _tiny.with_(name="rows_f32_noncausal", seed=4600),
    _tiny.with_(name="rows_f32_causal_ragged", N=1000, causal=True, seed=4700),
    _c64.with_(name="rows_bf16_d64_C32", N=2500, H_q=8, H_kv=4, d=64, C=32, K=5, segment=256, seed=4800),
    _tiny.with_(name="rows_bf16_G2_B2", B=2, N=777, H_q=4, H_kv=2, d=64, C=32, K=3, causal=True, dtype="bf16",
                seed=4900),
]


def _run(w, rows_per_head=None):
    dev = torch.device("cuda")
    x = workloads.prefill_inputs(w, device=dev)
    q, k = x["q"], x["k"]
    sel = api.select_exact(q, k, C=w.C, K=w.K, causal=w.causal)
    p = api.Prefill(api.Problem.of(q, k, C=w.C, K=w.K, causal=w.causal), dev)
    p(q, k, x["v"])
    pisa = p.sel
    torch.cuda.synchronize()
    rows = P.sample_rows(w, rows_per_head, extra_t=[t for (t, _) in x["needles"]])
    ref, gap = O.select_exact_rows(P.ocfg(w), P.host(q), P.host(k), rows)
    got = P.gather_rows(sel, rows)
    n, n_ex, bad, bad_ex = P.compare_selection(w, got, ref, gap)
    assert bad == 0, f"{w.name}: {bad} non-exempt mismatches of {n} rows ({n_ex} exempt)"
    # Output format: ascending, -1 padded, min(K, usable leaves) entries.
    for r, (b, h, t) in enumerate(rows):
        nv = min(w.K, (t // w.C + 1) if w.causal else -(-w.N // w.C))
        assert (got[r, :nv] >= 0).all() and (got[r, nv:] == -1).all()
        assert (np.diff(got[r, :nv]) > 0).all()
    # Recall of the pyramid search against the exact top K (reported).
    ps = P.gather_rows(pisa, rows)
    hit = sum(len(set(a[a >= 0]) & set(e[e >= 0])) for a, e in zip(ps, ref))
    tot = sum(int((e >= 0).sum()) for e in ref)
    return dict(rows=n, exempt=n_ex, exempt_mismatch=bad_ex, pisa_recall=hit / max(tot, 1))


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_exact_selector_parity_small(w):
    r = _run(w)
    print(w.name, r)


@pytest.mark.slow
@pytest.mark.parametrize("name,rows", [("needle_16k", 512), ("needle_256k", 96)])
def test_exact_selector_parity_full_size(name, rows):
    w = workloads.PREFILL[name]
    r = _run(w, rows)
    print(name, r)
