"""Paged-KV decode (mixed sequence lengths, one leaf block per page, pages in
shuffled order) through the C ABI, §Kernels (decoding) of the method's page.

* Oracle parity: each sequence's caches are read back through its block
  table, and its pyramid, selection and attention are compared with the fp64
  oracle on the prefix, at steps where sequences cross a leaf boundary and
  where the pyramid grows a new top level.
* The pyramid init and every fused step must also give bit-for-bit the
  dense-cache results on the same data, since both run the same arithmetic in
  the same order.
* A sequence whose next leaf has no page reports capacity and is skipped,
  like a full dense cache."""
import pytest
import torch

from hierarchical_top_block_mean_b200 import api, workloads
from test_parity_decode import _check_seq

pytestmark = pytest.mark.gpu

CASES = [
    workloads.DECODE["decode_64x128k"].with_(name="paged_C64_d128", S=5, context=900, steps=40, seed=7100),
    workloads.DECODE["decode_64x128k"].with_(name="paged_C32_d64_G4", S=4, context=300, steps=50, H_q=8, H_kv=2,
                                             d=64, C=32, K=5, seed=7200),
    workloads.DECODE["decode_64x128k"].with_(name="paged_G8_K16", S=3, context=700, steps=30, H_q=16, H_kv=2,
                                             seed=7300),
]


def _to_pages(w, kc, vc, lens, max_pages, gen):
    """Shuffled page pool holding every leaf a sequence may reach; returns
    k_pages, v_pages [P, H_kv, C, d] and the block table [S, max_pages]."""
    npages = w.S * max_pages + 3  # a few spare pages that no sequence uses
    perm = torch.randperm(npages, generator=gen, device="cpu")
    bt = perm[: w.S * max_pages].reshape(w.S, max_pages).to(torch.int32)
    kp = torch.zeros((npages, w.H_kv, w.C, w.d), dtype=kc.dtype, device=kc.device)
    vp = torch.zeros_like(kp)
    for s in range(w.S):
        for i in range(max_pages):
            kp[bt[s, i]] = kc[s, :, i * w.C:(i + 1) * w.C]
            vp[bt[s, i]] = vc[s, :, i * w.C:(i + 1) * w.C]
    return kp, vp, bt.to(kc.device)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_paged_decode_equals_dense(w):
    dev = torch.device("cuda")
    max_pages = -(-(w.context + w.steps) // w.C)
    cap = max_pages * w.C
    kc, vc, lens = workloads.decode_cache(w.with_(steps=cap - w.context), device=dev)
    lens -= torch.arange(w.S, device=dev, dtype=torch.int32) * 61  # mixed lengths
    gen = torch.Generator().manual_seed(w.seed)
    kp, vp, bt = _to_pages(w, kc, vc, lens, max_pages, gen)
    dense = api.DecodeState(S=w.S, cap=cap, H_q=w.H_q, H_kv=w.H_kv, d=w.d, C=w.C, K=w.K, dtype=w.torch_dtype,
                            device=dev, k_cache=kc, v_cache=vc, lens=lens.clone())
    paged = api.PagedDecodeState(S=w.S, max_pages=max_pages, H_q=w.H_q, H_kv=w.H_kv, d=w.d, C=w.C, K=w.K,
                                 k_pages=kp, v_pages=vp, block_table=bt, lens=lens.clone(), dtype=w.torch_dtype)
    dense.init()
    paged.init()
    torch.cuda.synchronize()
    assert torch.equal(dense.pyr, paged.pyr)
    for step in range(w.steps):
        q, k, v = workloads.decode_step_inputs(w, step, device=dev)
        dense.step(q, k, v)
        paged.step(q, k, v)
        torch.cuda.synchronize()
        assert torch.equal(dense.len, paged.len)
        assert torch.equal(dense.sel, paged.sel), step
        assert torch.equal(dense.out, paged.out), step
        assert torch.equal(dense.lse, paged.lse), step
    assert torch.equal(dense.pyr, paged.pyr)
    for s in range(w.S):
        n = int(dense.len[s])
        for i in range(-(-n // w.C)):
            m = min(w.C, n - i * w.C)
            assert torch.equal(paged.k_pages[bt[s, i], :, :m], dense.k_cache[s, :, i * w.C:i * w.C + m])
            assert torch.equal(paged.v_pages[bt[s, i], :, :m], dense.v_cache[s, :, i * w.C:i * w.C + m])
    assert int(dense.status) == 0 and int(paged.status) == 0


def test_paged_decode_missing_page_reports_capacity():
    w = CASES[1]
    dev = torch.device("cuda")
    max_pages = 12
    kc, vc, lens = workloads.decode_cache(w.with_(context=300, steps=max_pages * w.C - 300), device=dev)
    lens[:] = 320  # leaf 10 holds 0 keys; leaf 10 = the next token's leaf
    gen = torch.Generator().manual_seed(3)
    kp, vp, bt = _to_pages(w, kc, vc, lens, max_pages, gen)
    bt[1, 10] = -1  # sequence 1 has no page for its next leaf
    st = api.PagedDecodeState(S=w.S, max_pages=max_pages, H_q=w.H_q, H_kv=w.H_kv, d=w.d, C=w.C, K=w.K,
                              k_pages=kp, v_pages=vp, block_table=bt, lens=lens, dtype=w.torch_dtype)
    st.init()
    q, k, v = workloads.decode_step_inputs(w, 0, device=dev)
    st.step(q, k, v)
    torch.cuda.synchronize()
    assert int(st.status) == 4  # PISA_ERR_CAPACITY
    assert st.len.tolist() == [321, 320, 321, 321]


class _PagedView:
    """The attributes the decode oracle check reads, with each sequence's K and
    V caches gathered from its pages through the block table."""

    def __init__(self, st):
        S, mp, C = st.S, st.max_pages, st.C
        bt = st.block_table.long().clamp(min=0)
        self.k_cache = st.k_pages[bt].permute(0, 2, 1, 3, 4).reshape(S, st.H_kv, mp * C, st.d)
        self.v_cache = st.v_pages[bt].permute(0, 2, 1, 3, 4).reshape(S, st.H_kv, mp * C, st.d)
        self.len, self.cap, self.pyr = st.len, st.cap, st.pyr
        self.sel, self.out, self.lse = st.sel, st.out, st.lse


ORACLE_CASES = [
    # seq 0 grows 1000 -> 1040 tokens: leaf 15 fills and leaf 16 opens a new top level (M_1 16 -> 17)
    CASES[0].with_(name="paged_oracle_C64_G4", S=4, context=1000, steps=40, seed=7400),
    # C = 32: seq 0 grows 500 -> 530, crossing 512 tokens (M_1 16 -> 17)
    CASES[1].with_(name="paged_oracle_C32_G4", S=3, context=500, steps=30, seed=7500),
    # G_Q = 8, seq 1 (1024 - 61 = 963 tokens) crosses leaf 15 and seq 0 the new top level
    CASES[2].with_(name="paged_oracle_G8", S=3, context=1010, steps=24, seed=7600),
]


@pytest.mark.parametrize("w", ORACLE_CASES, ids=lambda w: w.name)
def test_paged_decode_matches_oracle(w):
    dev = torch.device("cuda")
    max_pages = -(-(w.context + w.steps) // w.C) + 1
    cap = max_pages * w.C
    kc, vc, lens = workloads.decode_cache(w.with_(steps=cap - w.context), device=dev)
    lens -= torch.arange(w.S, device=dev, dtype=torch.int32) * 61  # mixed lengths
    kp, vp, bt = _to_pages(w, kc, vc, lens, max_pages, torch.Generator().manual_seed(w.seed))
    st = api.PagedDecodeState(S=w.S, max_pages=max_pages, H_q=w.H_q, H_kv=w.H_kv, d=w.d, C=w.C, K=w.K,
                              k_pages=kp, v_pages=vp, block_table=bt, lens=lens, dtype=w.torch_dtype)
    st.init()
    start = lens.cpu()
    crossings = set()
    for step in range(w.steps):
        q, k, v = workloads.decode_step_inputs(w, step, device=dev)
        st.step(q, k, v)
        torch.cuda.synchronize()
        n_now = start + step + 1
        new_leaf = ((n_now - 1) % w.C == 0).any().item()
        new_level = any(api.pyramid_geometry(int(n), w.C)[0] > api.pyramid_geometry(int(n) - 1, w.C)[0]
                        for n in n_now.tolist() if n > 1)
        if new_leaf:
            crossings.add("leaf")
        if new_level:
            crossings.add("level")
        if step in (0, 1, w.steps - 1) or new_leaf or new_level or step % 8 == 0:
            view = _PagedView(st)
            for s in range(w.S):
                _check_seq(w, view, s, q)
    assert crossings == {"leaf", "level"}, crossings
    assert int(st.status) == 0
