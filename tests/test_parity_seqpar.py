"""Query shards of a sequence (sequence-parallel prefill) through the C ABI.

A shard's rows come from its own queries plus the whole sequence's keys,
values and pyramid. Its selection, output and lse must equal the same rows
of the whole-sequence run bit for bit, because a row's result depends on
nothing else (§TopK, §BSA). They must also match the oracle on sampled
rows. Shards start at arbitrary positions: a single first token, offsets that
are not leaf-aligned, a single last token. The cases cover every kernel
path: the tcgen05 leaf scorer (G_Q = 8, d = 128, C = 64), the mma.sync leaf
kernel (other bf16 shapes) and the fp32 row kernels. The full-size 256K
workload is checked split 8 ways. The sequence-parallel driver runs over a
one-rank NCCL group: its gather is then a copy, but it goes through the same
collective and stream waits."""
import numpy as np
import pytest
import torch
import torch.distributed as dist

import _parity as P
import oracle as O
from hierarchical_top_block_mean_b200 import api, seqpar, workloads

pytestmark = pytest.mark.gpu

CASES = [
    workloads.PREFILL["needle_256k"].with_(name="sp_G8_needle_4k", N=4100, n_needles=12, seed=9100),
    workloads.PREFILL["needle_16k"].with_(name="sp_G4_needle_3k", N=3000, n_needles=10, seed=9200),
    workloads.PREFILL["clustered_64k"].with_(name="sp_d64_C32_G2", N=2500, H_q=8, H_kv=4, d=64, C=32, K=5,
                                             segment=256, seed=9300),
    workloads.PREFILL["tiny_noncausal_1k"].with_(name="sp_f32_noncausal", seed=9400),
    workloads.PREFILL["tiny_noncausal_1k"].with_(name="sp_f32_causal", N=1000, causal=True, seed=9500),
    workloads.PREFILL["tiny_noncausal_1k"].with_(name="sp_bf16_G1_B2", B=2, N=900, H_q=2, H_kv=2, d=128, C=64, K=8,
                                                 causal=True, dtype="bf16", seed=9600),
]


def _bounds(N):
    """Shard boundaries: the first token alone, unaligned cuts, the last token alone."""
    return sorted({0, 1, 333, N // 2 + 7, N - 1, N})


def _whole(w, dev):
    x = workloads.prefill_inputs(w, device=dev)
    q, k, v = x["q"], x["k"], x["v"]
    p = api.Prefill(api.Problem.of(q, k, C=w.C, K=w.K, causal=w.causal), dev)
    p(q, k, v)
    return x, p


def _shard(w, p, q, k, v, a, b):
    qs = q[:, :, a:b].contiguous()
    sel = api.select_span(qs, k, p.pyr, q0=a, C=w.C, K=w.K, causal=w.causal)
    out, lse = api.sparse_attn_fwd_span(qs, k, v, sel, q0=a, C=w.C, causal=w.causal)
    return sel, out, lse


def _assert_rows_equal(name, p, a, b, sel, out, lse):
    assert torch.equal(sel, p.sel[:, :, a:b]), f"{name} [{a}, {b}): selection differs from the whole run"
    assert torch.equal(out, p.out[:, :, a:b]), f"{name} [{a}, {b}): output differs from the whole run"
    assert torch.equal(lse, p.lse[:, :, a:b]), f"{name} [{a}, {b}): lse differs from the whole run"


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_query_shards_equal_whole_sequence_rows(w):
    dev = torch.device("cuda")
    x, p = _whole(w, dev)
    q, k, v = x["q"], x["k"], x["v"]
    bounds = _bounds(w.N)
    shards = [(a, b, *_shard(w, p, q, k, v, a, b)) for a, b in zip(bounds[:-1], bounds[1:])]
    torch.cuda.synchronize()
    for a, b, sel, out, lse in shards:
        _assert_rows_equal(w.name, p, a, b, sel, out, lse)
    # The oracle on sampled rows of the unaligned middle shard, read from the shard's own arrays.
    a, b, sel, out, lse = shards[2]
    rng = np.random.default_rng(w.seed)
    ts = np.unique(np.concatenate([[a, b - 1], rng.integers(a, b, size=48)]))
    rows = np.array([(bb, h, t) for bb in range(w.B) for h in range(w.H_kv) for t in ts], dtype=np.int64)
    local = rows.copy()
    local[:, 2] -= a
    qh, kh, vh = P.host(q), P.host(k), P.host(v)
    cfg = P.ocfg(w)
    pyr_ref = P.check_pyramid(w, kh, P.host(p.pyr))
    sel_ref, gap = O.select_rows(cfg, qh, kh, pyr_ref, rows)
    sel_gpu = P.gather_rows(sel, local)
    n, _, bad, _ = P.compare_selection(w, sel_gpu, sel_ref, gap)
    assert bad == 0, f"{w.name}: shard [{a}, {b}) has {bad} selection mismatches of {n}"
    out_ref, lse_ref = O.attn_rows(cfg, qh, kh, vh, rows, sel_gpu)
    P.check_attention(w, P.gather_out(w, out, local), P.gather_lse(w, lse, local), out_ref, lse_ref)


@pytest.mark.slow
def test_full_size_eight_shards():
    w = workloads.PREFILL["needle_256k"]
    dev = torch.device("cuda")
    x, p = _whole(w, dev)
    q, k, v = x["q"], x["k"], x["v"]
    for r in range(8):
        a, n = seqpar.shard_span(w.N, 8, r)
        sel, out, lse = _shard(w, p, q, k, v, a, a + n)
        torch.cuda.synchronize()
        _assert_rows_equal(w.name, p, a, a + n, sel, out, lse)
        del sel, out, lse


def test_driver_over_one_rank_nccl_group():
    w = CASES[0]
    dev = torch.device("cuda", torch.cuda.current_device())
    x, p = _whole(w, dev)
    q, k, v = x["q"], x["k"], x["v"]
    own = not dist.is_initialized()
    if own:
        dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1, device_id=dev)
    try:
        sp = seqpar.SeqParallelPrefill(api.Problem.of(q, k, C=w.C, K=w.K, causal=w.causal), device=dev)
        assert (sp.q0, sp.n) == (0, w.N)
        out, lse, sel = sp(q, k, v)
        torch.cuda.synchronize()
        assert torch.equal(sp.k_full, k) and torch.equal(sp.v_full, v) and torch.equal(sp.shard.pyr, p.pyr)
        _assert_rows_equal(w.name, p, 0, w.N, sel, out, lse)
        with pytest.raises(ValueError):
            sp(q[:, :, :-1].contiguous(), k, v)
    finally:
        if own:
            dist.destroy_process_group()
