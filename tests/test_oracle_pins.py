"""Pins for the fp64 CPU oracle, checked against what the pages and the
mathematics fix, never against the oracle itself.

Page citations name sections of the hyper.ai page of "Block Sparse Attention
with Log-Linear Complexity":
  §BSA     block-sparse attention equation
  §Pyramid level sizes, Concat, mean-pooled summaries
  §TopK    coarse-to-fine candidate sets, keep-all rule, LSE block score
  §Kernels GQA sum of scores; decode pyramid update

Each pin is chosen so that a plausible mistake in the oracle (a dropped head,
a wrong child index, a wrong sign, a missing causal mask, an off-by-one block
span, an ancestor not updated) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from hierarchical_top_block_mean_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cfg(o, w, **kw):
    return o.make_cfg(B=w.B, N=w.N, H_q=w.H_q, H_kv=w.H_kv, d=w.d, C=w.C, K=w.K, causal=w.causal,
                      dtype_code=0 if w.dtype == "f32" else 1, **kw)


def _small(name="pin", **kw):
    base = dict(B=1, N=512, H_q=4, H_kv=2, d=16, C=16, K=4, causal=True, dtype="f32", seed=77)
    base.update(kw)
    return workloads.Prefill(name, **base)


def _dense_pool(k64: torch.Tensor, span: int) -> torch.Tensor:
    """Direct average of raw keys over consecutive spans (full spans only),
    via avg_pool1d: [B,H,N,d] -> [B,H,N/span,d]."""
    B, H, N, d = k64.shape
    x = k64.permute(0, 1, 3, 2).reshape(B * H, d, N)
    y = F.avg_pool1d(x, kernel_size=span, stride=span)
    return y.reshape(B, H, d, -1).permute(0, 1, 3, 2)


# ---------------------------------------------------------------- geometry

def _golden_geometry():
    rows = []
    with open(os.path.join(GOLDEN, "geometry.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            a, b, c = line.split("|")
            N, C = map(int, a.split())
            rows.append((N, C, list(map(int, b.split())), int(c)))
    return rows


@pytest.mark.parametrize("N,C,M,R", _golden_geometry())
def test_geometry_golden(oracle, N, C, M, R):
    sizes, offs = oracle.geometry(N, C)
    assert sizes[0] == N
    assert list(sizes[1:]) == M
    assert offs[-1] == R
    assert list(offs) == [0] + list(np.cumsum(M))


@pytest.mark.parametrize("m", range(0, 15))
def test_geometry_power_of_two_closed_form(oracle, m):
    # M_1 = 2^m leaves: L = m + 1 levels, level l has 2^(m-l+1) blocks, R = 2^(m+1) - 1.
    sizes, offs = oracle.geometry(64 << m, 64)
    assert len(sizes) - 1 == m + 1
    assert list(sizes[1:]) == [2 ** (m - l + 1) for l in range(1, m + 2)]
    assert offs[-1] == 2 ** (m + 1) - 1


# ----------------------------------------------------------------- pyramid

def test_pyramid_ragged_golden(oracle):
    with open(os.path.join(GOLDEN, "pyramid_ragged.txt")) as f:
        cases = [l for l in f if l.strip() and not l.startswith("#")]
    assert cases
    for line in cases:
        a, b, c = line.split("|")
        keys = np.array(list(map(float, a.split())), np.float32).reshape(1, 1, -1, 1)
        C = int(b)
        want = np.array(list(map(float, c.split())))
        got = oracle.build_pyramid(keys, C).reshape(-1)
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_pyramid_equals_direct_span_average(oracle, dtype):
    # N = C * 2^5: every block at every level is full, so level l equals the
    # plain average of the raw keys over spans of C * 2^(l-1) (§Pyramid).
    w = _small(N=32 * 16, C=16, d=8, H_kv=3, H_q=3, dtype=dtype, B=2)
    x = workloads.prefill_inputs(w)
    pyr = oracle.build_pyramid(x["k"], w.C)
    sizes, offs = oracle.geometry(w.N, w.C)
    k64 = x["k"].double()
    for l in range(1, len(sizes)):
        want = _dense_pool(k64, w.C << (l - 1)).numpy()
        got = pyr[:, :, offs[l - 1]:offs[l], :]
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


# -------------------------------------------------------------- selection

def _trace(oracle, w, x, rows):
    cfg = _cfg(oracle, w)
    pyr = oracle.build_pyramid(x["k"], w.C)
    sel, gap, tr = oracle.select_rows(cfg, x["q"], x["k"], pyr, rows, trace=True)
    return cfg, pyr, sel, gap, tr


def _dense_leaf_lse(x, w, b, h, t, i):
    """Exact raw-key block LSE summed over the GQA group, via torch.logsumexp."""
    G = w.H_q // w.H_kv
    q = x["q"][b, h * G:(h + 1) * G, t, :].double()
    lo, hi = i * w.C, min((i + 1) * w.C, w.N)
    if w.causal:
        hi = min(hi, t + 1)
    k = x["k"][b, h, lo:hi, :].double()
    s = (q @ k.T) / math.sqrt(w.d)
    return torch.logsumexp(s, dim=1).sum().item()


def test_leaf_score_is_exact_block_lse(oracle):
    # §TopK: at the leaf level the children are the raw keys, so the score is
    # the exact block LSE; §Kernels: summed over the query heads of the group.
    w = _small(N=1000, C=16, K=4, causal=True)  # ragged last leaf (1000 = 62*16 + 8)
    x = workloads.prefill_inputs(w)
    rows = [(0, h, t) for h in range(w.H_kv) for t in (70, 200, 511, 777, 999)]
    _, _, _, _, tr = _trace(oracle, w, x, rows)
    checked = 0
    for r, (b, h, t) in enumerate(rows):
        n = tr["n"][r, 1]
        assert n > w.K  # leaf level scored for these rows
        for s in range(n):
            i = tr["cand"][r, 1, s]
            want = _dense_leaf_lse(x, w, b, h, t, i)
            assert abs(tr["score"][r, 1, s] - want) < 1e-9
            checked += 1
    assert checked > 50


def test_inner_level_scores_from_direct_averages(oracle):
    # §TopK inner-level score: LSE over the (at most g) child summaries, summed
    # over the group. With full blocks the child summaries are plain span
    # averages (avg_pool1d) and the LSE a torch.logsumexp over the pair.
    w = _small(N=1024, C=16, K=3, causal=False, H_q=6, H_kv=2)
    x = workloads.prefill_inputs(w)
    rows = [(0, h, t) for h in range(2) for t in (0, 313, 1023)]
    _, _, _, _, tr = _trace(oracle, w, x, rows)
    G = w.H_q // w.H_kv
    k64 = x["k"].double()
    n_checked = 0
    for r, (b, h, t) in enumerate(rows):
        for l in range(2, tr["n"].shape[1]):
            n = tr["n"][r, l]
            if n <= w.K:
                assert np.isnan(tr["score"][r, l, :n]).all()
                continue
            child = _dense_pool(k64, w.C << (l - 2))[b, h]  # level l-1 summaries
            q = x["q"][b, h * G:(h + 1) * G, t, :].double()
            logits = (q @ child.T) / math.sqrt(w.d)  # [G, M_{l-1}]
            for s in range(n):
                i = tr["cand"][r, l, s]
                want = torch.logsumexp(logits[:, 2 * i:2 * i + 2], dim=1).sum().item()
                assert abs(tr["score"][r, l, s] - want) < 1e-9
                n_checked += 1
    assert n_checked > 20


def test_inner_level_causal_scores_leave_out_later_children(oracle):
    # §TopK inner-level score under the causal reading: a candidate block
    # whose first key is <= t is usable, but its second child may start after
    # t; that child's summary must not enter the LSE. The summaries themselves
    # stay the static whole-block means of §Pyramid (avg_pool1d here), so only
    # the set of children changes. A filter applied at the leaf level alone
    # fails this pin.
    w = _small(N=2048, C=16, K=3, causal=True, H_q=6, H_kv=2, d=16, seed=31)
    x = workloads.prefill_inputs(w)
    rng = np.random.default_rng(17)
    rows = [(0, h, int(t)) for h in range(w.H_kv) for t in rng.integers(4 * w.C, w.N, 120)]
    _, _, _, _, tr = _trace(oracle, w, x, rows)
    sizes, _ = oracle.geometry(w.N, w.C)
    G = w.H_q // w.H_kv
    k64 = x["k"].double()
    straddling = 0
    for r, (b, h, t) in enumerate(rows):
        q = x["q"][b, h * G:(h + 1) * G, t, :].double()
        for l in range(2, len(sizes)):
            n = tr["n"][r, l]
            if n <= w.K:
                continue
            child_span = w.C << (l - 2)
            child = _dense_pool(k64, child_span)[b, h]  # static level l-1 means
            for s in range(n):
                i = tr["cand"][r, l, s]
                kids = [c for c in (2 * i, 2 * i + 1) if c < sizes[l - 1] and c * child_span <= t]
                assert kids and kids[0] == 2 * i
                straddling += len(kids) == 1 and 2 * i + 1 < sizes[l - 1]
                logits = (q @ child[kids].T) / math.sqrt(w.d)  # [G, |kids|]
                want = torch.logsumexp(logits, dim=1).sum().item()
                assert abs(tr["score"][r, l, s] - want) < 1e-9
    assert straddling > 50


@pytest.mark.parametrize("causal", [False, True])
def test_exact_ties_break_toward_lower_block_index(oracle, causal):
    # Tie rule (the pages leave it open; read as: equal scores go to the lower
    # block index). When every key is the same vector v, every full block of
    # every level has the same summary v, so all full candidates tie exactly:
    # a block's LSE over n equal logits is s + log n. A block cut by the causal
    # limit has fewer usable children and scores strictly lower. Every level
    # therefore keeps the K lowest full blocks, whose children are again the
    # lowest, and the selection is exactly leaves 0..K-1 for every query that
    # can see more than K leaves; the flat and exact selectors agree.
    w = _small(N=1024, C=16, K=4, causal=causal, H_q=4, H_kv=2, d=16, seed=41)
    x = workloads.prefill_inputs(w)
    vec = torch.randn(w.d, generator=torch.Generator().manual_seed(2))
    k = vec.expand(w.B, w.H_kv, w.N, w.d).contiguous()
    cfg = _cfg(oracle, w)
    pyr = oracle.build_pyramid(k, w.C)
    ts = [t for t in range(0, w.N, 11) if t // w.C + 1 > w.K]
    rows = [(0, h, t) for h in range(w.H_kv) for t in ts]
    want = np.tile(np.arange(w.K, dtype=np.int32), (len(rows), 1))
    sel, gap = oracle.select_rows(cfg, x["q"], k, pyr, rows)
    assert np.array_equal(sel, want)
    # The K-th and (K+1)-th candidates tie at some level, except causal rows
    # whose only scored level holds K full leaves and the cut one.
    assert (gap >= 0).all() and (gap == 0).mean() > (0.999 if not causal else 0.9)
    s_flat, _ = oracle.select_flat_rows(cfg, x["q"], pyr, rows)
    s_exact, _ = oracle.select_exact_rows(cfg, x["q"], k, rows)
    assert np.array_equal(s_flat, want)
    assert np.array_equal(s_exact, want)


def test_kept_sets_follow_score_then_lower_index_on_recurring_blocks(oracle):
    # With leaf contents that recur with period 3, blocks of equal content at
    # every level have identical summaries, so many candidates tie exactly and
    # the K-th place often falls inside a tied class. At every scored level the
    # kept set must be the first K candidates when ordered by score (higher
    # first) and then by block index (lower first).
    w = _small(N=3000, C=16, K=5, causal=True, H_q=4, H_kv=2, d=16, seed=43, structure="periodic", period=3)
    x = workloads.prefill_inputs(w)
    rows = [(0, h, t) for h in range(w.H_kv) for t in range(100, w.N, 13)]
    _, _, _, _, tr = _trace(oracle, w, x, rows)
    tied_at_k = 0
    for r in range(len(rows)):
        for l in range(1, tr["n"].shape[1]):
            n = tr["n"][r, l]
            if n <= w.K:
                continue
            cand = tr["cand"][r, l, :n]
            sc = tr["score"][r, l, :n]
            order = sorted(range(n), key=lambda m: (-sc[m], cand[m]))
            want = {int(cand[m]) for m in order[: w.K]}
            got = {int(c) for c, kk in zip(cand, tr["kept"][r, l, :n]) if kk}
            assert got == want
            tied_at_k += sc[order[w.K - 1]] == sc[order[w.K]]
    assert tied_at_k > 100


@pytest.mark.parametrize("causal", [False, True])
def test_large_K_selects_everything_and_attention_is_dense(oracle, causal):
    # With K >= number of leaves nothing is ever scored (§TopK keep-all rule),
    # so every valid block is selected and block-sparse attention is dense
    # attention (torch SDPA in fp64).
    w = _small(N=300, C=16, K=19, causal=causal, H_q=4, H_kv=2, d=16)  # 19 leaves, ragged
    x = workloads.prefill_inputs(w)
    cfg = _cfg(oracle, w)
    pyr = oracle.build_pyramid(x["k"], w.C)
    rows = [(0, h, t) for h in range(w.H_kv) for t in range(w.N)]
    sel, gap = oracle.select_rows(cfg, x["q"], x["k"], pyr, rows)
    for r, (b, h, t) in enumerate(rows):
        nv = (t // w.C + 1) if causal else 19
        assert list(sel[r]) == list(range(nv)) + [-1] * (w.K - nv)
        assert math.isinf(gap[r])
    out, lse = oracle.attn_rows(cfg, x["q"], x["k"], x["v"], rows, sel)
    q = x["q"].double()
    k = x["k"].double().repeat_interleave(2, dim=1)
    v = x["v"].double().repeat_interleave(2, dim=1)
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=causal)  # [1, H_q, N, d]
    got = torch.from_numpy(out).reshape(w.H_kv, w.N, 2, w.d).permute(0, 2, 1, 3).reshape(1, w.H_q, w.N, w.d)
    assert torch.allclose(got, ref, atol=1e-12, rtol=0)
    s = (q @ k.transpose(-1, -2)) / math.sqrt(w.d)
    if causal:
        s = s.masked_fill(torch.ones(w.N, w.N, dtype=torch.bool).triu(1), float("-inf"))
    lref = torch.logsumexp(s, -1)
    lgot = torch.from_numpy(lse).reshape(w.H_kv, w.N, 2).permute(0, 2, 1).reshape(1, w.H_q, w.N)
    assert torch.allclose(lgot, lref, atol=1e-12, rtol=0)


@pytest.mark.parametrize("causal", [False, True])
def test_attention_on_arbitrary_selection_matches_masked_sdpa(oracle, causal):
    # §BSA: attention over the raw keys of the selected blocks only.
    w = _small(N=200, C=16, K=5, causal=causal, H_q=6, H_kv=3, d=32)
    x = workloads.prefill_inputs(w)
    cfg = _cfg(oracle, w)
    g = torch.Generator().manual_seed(5)
    rows = [(0, h, t) for h in range(w.H_kv) for t in range(0, w.N, 7)]
    M1 = (w.N + w.C - 1) // w.C
    sel = np.full((len(rows), w.K), -1, np.int32)
    for r, (b, h, t) in enumerate(rows):
        nv = (t // w.C + 1) if causal else M1
        pick = torch.randperm(nv, generator=g)[: min(w.K - 1, nv)].tolist()
        if causal and (t // w.C) not in pick and len(pick) < w.K:
            pick.append(t // w.C)
        pick = sorted(pick)
        sel[r, : len(pick)] = pick
    out, lse = oracle.attn_rows(cfg, x["q"], x["k"], x["v"], rows, sel)
    G = w.H_q // w.H_kv
    for r, (b, h, t) in enumerate(rows):
        mask = torch.zeros(w.N, dtype=torch.bool)
        for i in sel[r]:
            if i >= 0:
                mask[i * w.C:(i + 1) * w.C] = True
        if causal:
            mask[t + 1:] = False
        q = x["q"][b, h * G:(h + 1) * G, t:t + 1, :].double()
        k = x["k"][b, h].double().unsqueeze(0).expand(G, -1, -1)
        v = x["v"][b, h].double().unsqueeze(0).expand(G, -1, -1)
        ref = F.scaled_dot_product_attention(q, k, v, attn_mask=mask.view(1, 1, -1).expand(G, 1, -1))
        np.testing.assert_allclose(out[r], ref[:, 0, :].numpy(), atol=1e-12, rtol=0)


def test_selection_invariants(oracle):
    # §TopK: |A^{(l-1)}| <= gK; kept sets are subsets of the valid
    # candidates; each level's candidates are children of the previous kept
    # blocks; |T| = min(K, #valid leaves); T is valid, ascending, -1 padded.
    w = _small(N=2000, C=8, K=5, causal=True, H_q=4, H_kv=2, d=16)
    x = workloads.prefill_inputs(w)
    rows = [(0, h, t) for h in range(2) for t in range(0, w.N, 3)]
    _, _, sel, gap, tr = _trace(oracle, w, x, rows)
    sizes, _ = oracle.geometry(w.N, w.C)
    L = len(sizes) - 1
    for r, (b, h, t) in enumerate(rows):
        prev_kept = None
        for l in range(L, 0, -1):
            n = tr["n"][r, l]
            assert n <= 2 * w.K
            cand = list(tr["cand"][r, l, :n])
            span = w.C << (l - 1)
            assert all(0 <= i < sizes[l] and i * span <= t for i in cand)
            if prev_kept is not None:
                kids = {c for p in prev_kept for c in (2 * p, 2 * p + 1)}
                assert set(cand) <= kids
                # every valid child of a kept block is a candidate
                assert {c for c in kids if c < sizes[l] and c * span <= t} == set(cand)
            kept = [i for i, kk in zip(cand, tr["kept"][r, l, :n]) if kk]
            assert len(kept) == min(n, w.K)
            prev_kept = kept
        nv = min(w.K, t // w.C + 1)
        s = list(sel[r])
        assert s[:nv] == sorted(prev_kept) and all(v == -1 for v in s[nv:])
        assert len(set(s[:nv])) == nv


def test_first_scored_level_sees_all_valid_blocks(oracle):
    # Starting at the root and keeping every level with <= K valid blocks
    # unscored means the first scored level's candidates are exactly all valid
    # blocks of that level (the device kernels start there).
    w = _small(N=4096, C=16, K=6, causal=True)
    x = workloads.prefill_inputs(w)
    rows = [(0, h, t) for h in range(2) for t in range(0, w.N, 37)]
    _, _, _, _, tr = _trace(oracle, w, x, rows)
    sizes, _ = oracle.geometry(w.N, w.C)
    for r, (_, _, t) in enumerate(rows):
        for l in range(len(sizes) - 1, 0, -1):
            n = tr["n"][r, l]
            nv = min(sizes[l], t // (w.C << (l - 1)) + 1)
            if n > w.K:
                assert list(tr["cand"][r, l, :n]) == list(range(nv))
                break
            assert n == nv


@pytest.mark.parametrize("causal", [False, True])
def test_greedy_descent_finds_planted_leaf(oracle, causal):
    # K = 1 makes the selection a greedy root-to-leaf descent: every level
    # keeps the single best block. A leaf whose keys all equal a large
    # multiple of the query direction dominates its ancestors' mean summaries
    # at every level, so the descent must end on exactly that leaf. A wrong
    # child index, a reversed sort or a dropped level fails this.
    N, C, d = 1024, 8, 16
    w = _small(N=N, C=C, d=d, K=1, causal=causal, H_q=2, H_kv=1)
    x = workloads.prefill_inputs(w)
    t = N - 1
    qdir = x["q"][0, :, t, :].sum(0)
    qdir = qdir / qdir.norm()
    cfg = _cfg(oracle, w)
    for j in [0, 1, 2, 5, 64, 101, 127]:
        k = x["k"].clone() * 0.05
        k[0, 0, j * C:(j + 1) * C, :] = 40.0 * qdir
        pyr = oracle.build_pyramid(k, C)
        sel, _ = oracle.select_rows(cfg, x["q"], k, pyr, [(0, 0, t)])
        assert list(sel[0]) == [j]


def test_unscored_keep_rule_early_queries(oracle):
    # §TopK: when a level has at most K valid candidates all are kept without
    # scoring; for early causal queries that reaches the leaves.
    w = _small(N=1024, C=16, K=5, causal=True)
    x = workloads.prefill_inputs(w)
    cfg = _cfg(oracle, w)
    pyr = oracle.build_pyramid(x["k"], w.C)
    rows = [(0, 1, t) for t in range(0, 5 * 16)]
    sel, gap = oracle.select_rows(cfg, x["q"], x["k"], pyr, rows)
    for r, (_, _, t) in enumerate(rows):
        nv = t // 16 + 1
        assert list(sel[r]) == list(range(nv)) + [-1] * (5 - nv)
        assert math.isinf(gap[r])


def test_gap_is_kth_minus_next_score(oracle):
    w = _small(N=2048, C=16, K=4, causal=True)
    x = workloads.prefill_inputs(w)
    rows = [(0, h, t) for h in range(2) for t in range(300, 2048, 97)]
    _, _, _, gap, tr = _trace(oracle, w, x, rows)
    for r in range(len(rows)):
        g = math.inf
        for l in range(tr["n"].shape[1]):
            n = tr["n"][r, l]
            if n > w.K:
                s = np.sort(tr["score"][r, l, :n])[::-1]
                g = min(g, s[w.K - 1] - s[w.K])
        assert gap[r] == pytest.approx(g, abs=1e-12)


def test_planted_needles_are_found(oracle):
    # Structure check (not a parity condition): a leaf whose keys point along
    # the group's query direction is selected for that query in nearly every
    # case. A sign error or a dropped head would lose most needles.
    w = workloads.Prefill("needle_small", B=1, N=4096, H_q=8, H_kv=2, d=64, C=32, K=4, causal=True,
                          dtype="bf16", structure="needle", n_needles=24, seed=11)
    x = workloads.prefill_inputs(w)
    cfg = _cfg(oracle, w)
    pyr = oracle.build_pyramid(x["k"], w.C)
    rows = [(0, h, t) for (t, j) in x["needles"] for h in range(w.H_kv)]
    sel, _ = oracle.select_rows(cfg, x["q"], x["k"], pyr, rows)
    want = [j for (t, j) in x["needles"] for h in range(w.H_kv)]
    hits = sum(int(j in list(s)) for s, j in zip(sel, want))
    assert hits >= 0.9 * len(rows)


# ------------------------------------------------------------------- flat

@pytest.mark.parametrize("causal", [False, True])
def test_flat_selector_is_topk_of_dense_summary_scores(oracle, causal):
    # Flat scoring of all M = ceil(N/C) leaf summaries (§BSA): a dense fp64
    # matmul of each query head with the avg-pooled leaf summaries, summed
    # over the group, then the K largest (torch.topk).
    w = _small(N=1024, C=16, K=6, causal=causal, H_q=6, H_kv=2, d=32)
    x = workloads.prefill_inputs(w)
    cfg = _cfg(oracle, w)
    pyr = oracle.build_pyramid(x["k"], w.C)
    rows = [(0, h, t) for h in range(2) for t in range(0, w.N, 5)]
    sel, gap = oracle.select_flat_rows(cfg, x["q"], pyr, rows)
    leaves = _dense_pool(x["k"].double(), w.C)[0]  # [H_kv, 64, d]
    G = w.H_q // w.H_kv
    for r, (b, h, t) in enumerate(rows):
        q = x["q"][b, h * G:(h + 1) * G, t, :].double()
        u = (q @ leaves[h].T / math.sqrt(w.d)).sum(0)
        nv = (t // w.C + 1) if causal else u.numel()
        if nv <= w.K:
            want = list(range(nv))
        else:
            want = sorted(torch.topk(u[:nv], w.K).indices.tolist())
        assert list(sel[r][: len(want)]) == want


# ------------------------------------------------------------ exact flat

def _dense_block_lse_scores(x, w, b, h, t):
    """All leaves' exact scores for one row from the dense score matrix: the
    [G, N] logits of the group's heads (fp64), masked causally, split into
    C-wide blocks (the ragged last one padded with -inf), logsumexp per block
    (torch.logsumexp), summed over the heads."""
    G = w.H_q // w.H_kv
    q = x["q"][b, h * G:(h + 1) * G, t, :].double()
    k = x["k"][b, h].double()
    s = (q @ k.T) / math.sqrt(w.d)
    if w.causal:
        s[:, t + 1:] = -math.inf
    M1 = -(-w.N // w.C)
    pad = torch.full((G, M1 * w.C - w.N), -math.inf, dtype=s.dtype)
    blocks = torch.cat([s, pad], dim=1).reshape(G, M1, w.C)
    u = torch.logsumexp(blocks, dim=2).sum(0)
    nv = (t // w.C + 1) if w.causal else M1
    return u[:nv]


@pytest.mark.parametrize("causal", [False, True])
def test_exact_selector_is_topk_of_dense_block_lse(oracle, causal):
    # Exact single-level selection (§BSA scoring every block, with §TopK's LSE
    # block score): the K largest dense block LSEs (torch.topk), ragged last
    # leaf included (N = 1000 = 62 * 16 + 8).
    w = _small(N=1000, C=16, K=5, causal=causal, H_q=6, H_kv=2, d=32, seed=5)
    x = workloads.prefill_inputs(w)
    cfg = _cfg(oracle, w)
    rows = [(0, h, t) for h in range(2) for t in range(0, w.N, 7)]
    sel, gap = oracle.select_exact_rows(cfg, x["q"], x["k"], rows)
    for r, (b, h, t) in enumerate(rows):
        u = _dense_block_lse_scores(x, w, b, h, t)
        if u.numel() <= w.K:
            want = list(range(u.numel()))
            assert gap[r] == math.inf
        else:
            top = torch.topk(u, w.K + 1)
            want = sorted(top.indices[: w.K].tolist())
            assert gap[r] == pytest.approx((top.values[w.K - 1] - top.values[w.K]).item(), abs=1e-9)
        assert list(sel[r][: len(want)]) == want
        assert all(v == -1 for v in sel[r][len(want):])


def test_exact_selector_equals_pyramid_when_every_leaf_is_scored(oracle):
    # With M_2 <= K < M_1 the coarse-to-fine search starts at the leaf level
    # and scores every usable leaf, so it must return the exact selection.
    w = _small(N=512, C=16, K=16, causal=True, H_q=4, H_kv=2, d=16, seed=9)  # M_1 = 32, M_2 = 16
    x = workloads.prefill_inputs(w)
    cfg = _cfg(oracle, w)
    pyr = oracle.build_pyramid(x["k"], w.C)
    rows = [(0, h, t) for h in range(2) for t in range(0, w.N, 3)]
    s_pyr, _ = oracle.select_rows(cfg, x["q"], x["k"], pyr, rows)
    s_ex, _ = oracle.select_exact_rows(cfg, x["q"], x["k"], rows)
    assert np.array_equal(s_pyr, s_ex)


def test_exact_selector_finds_planted_needles(oracle):
    w = workloads.Prefill("needle_small", B=1, N=4096, H_q=8, H_kv=2, d=64, C=32, K=4, causal=True,
                          dtype="bf16", structure="needle", n_needles=24, seed=11)
    x = workloads.prefill_inputs(w)
    cfg = _cfg(oracle, w)
    rows = [(0, h, t) for (t, j) in x["needles"] for h in range(w.H_kv)]
    sel, _ = oracle.select_exact_rows(cfg, x["q"], x["k"], rows)
    want = [j for (t, j) in x["needles"] for h in range(w.H_kv)]
    assert all(j in list(s) for s, j in zip(sel, want))


# --------------------------------------------------------------- backward

def _random_selection(w, rng):
    """A valid selection [B, H_kv, N, K]: up to K distinct usable leaves per
    row (some rows get fewer), ascending, -1 padded."""
    M1 = -(-w.N // w.C)
    sel = np.full((w.B, w.H_kv, w.N, w.K), -1, np.int32)
    for b in range(w.B):
        for h in range(w.H_kv):
            for t in range(w.N):
                nv = (t // w.C + 1) if w.causal else M1
                m = int(rng.integers(1, min(w.K, nv) + 1))
                sel[b, h, t, :m] = np.sort(rng.choice(nv, m, replace=False))
    return sel


@pytest.mark.parametrize("causal", [False, True])
def test_attention_backward_matches_autograd(oracle, causal):
    # Gradient of §BSA's attention over a fixed selection: torch autograd
    # (fp64) through dense attention whose mask admits exactly the selected
    # blocks' keys (and, causally, keys <= t); the GQA key/value sharing is a
    # repeat over the group, so autograd sums the group's contributions.
    w = _small(N=200, C=16, K=3, causal=causal, H_q=6, H_kv=2, d=16, seed=21)
    x = workloads.prefill_inputs(w)
    rng = np.random.default_rng(3)
    sel = _random_selection(w, rng)
    g = torch.randn(w.B, w.H_q, w.N, w.d, generator=torch.Generator().manual_seed(4))
    dq, dk, dv = oracle.attn_bwd(_cfg(oracle, w), x["q"], x["k"], x["v"], sel, g)
    G = w.H_q // w.H_kv
    q = x["q"].double().requires_grad_()
    k = x["k"].double().requires_grad_()
    v = x["v"].double().requires_grad_()
    allowed = torch.zeros(w.B, w.H_kv, w.N, w.N, dtype=torch.bool)
    for b in range(w.B):
        for h in range(w.H_kv):
            for t in range(w.N):
                for i in sel[b, h, t]:
                    if i >= 0:
                        allowed[b, h, t, i * w.C:(i + 1) * w.C] = True
    if causal:
        allowed &= torch.ones(w.N, w.N, dtype=torch.bool).tril()
    mask = allowed.repeat_interleave(G, dim=1)
    s = (q @ k.repeat_interleave(G, 1).transpose(-1, -2)) / math.sqrt(w.d)
    p = torch.softmax(s.masked_fill(~mask, -math.inf), dim=-1)
    o = p @ v.repeat_interleave(G, 1)
    (o * g.double()).sum().backward()
    for got, want in ((dq, q.grad), (dk, k.grad), (dv, v.grad)):
        assert np.abs(got - want.numpy()).max() < 1e-10


def test_attention_backward_dq_rows_match_all_rows(oracle):
    # A row's dq depends on that row alone: the per-row entry point (used for
    # sampled rows at full size) must reproduce the all-rows gradient.
    w = _small(N=150, C=16, K=3, causal=True, H_q=4, H_kv=2, d=16, seed=23)
    x = workloads.prefill_inputs(w)
    sel = _random_selection(w, np.random.default_rng(5))
    g = torch.randn(w.B, w.H_q, w.N, w.d, generator=torch.Generator().manual_seed(6))
    dq, _, _ = oracle.attn_bwd(_cfg(oracle, w), x["q"], x["k"], x["v"], sel, g)
    rows = [(0, h, t) for h in range(w.H_kv) for t in range(0, w.N, 7)]
    got = oracle.attn_bwd_dq_rows(_cfg(oracle, w), x["q"], x["k"], x["v"], rows,
                                  np.stack([sel[b, h, t] for (b, h, t) in rows]), g)
    G = w.H_q // w.H_kv
    for r, (b, h, t) in enumerate(rows):
        assert np.abs(got[r] - dq[b, h * G:(h + 1) * G, t]).max() < 1e-12


# ------------------------------------------------------------------ decode

def test_decode_incremental_pyramid_equals_batch(oracle):
    # §Kernels (decoding): caching the mean pyramid and, per new token,
    # updating only the current leaf and its ancestors must reproduce the
    # pyramid built from scratch over the prefix, including ragged leaves and
    # the moments a new top level appears.
    C, d, cap = 4, 3, 75
    g = torch.Generator().manual_seed(3)
    keys = torch.randn(cap, d, generator=g).to(torch.bfloat16)
    sizes_c, offs_c = oracle.geometry(cap, C)
    pyr = np.zeros((offs_c[-1], d), np.float64)
    for n in range(cap):
        oracle.decode_append(keys, n, C, cap, pyr)
        want = oracle.build_pyramid(keys[: n + 1].reshape(1, 1, n + 1, d), C)[0, 0]
        sizes, offs = oracle.geometry(n + 1, C)
        for l in range(1, len(sizes)):
            got = pyr[offs_c[l - 1]:offs_c[l - 1] + sizes[l]]
            np.testing.assert_allclose(got, want[offs[l - 1]:offs[l]], rtol=0, atol=1e-12)


def test_decode_query_sees_every_block(oracle):
    # The new token is the last position, so under the causal reading every
    # block of the prefix is valid; the selection equals the non-causal one on
    # the same prefix.
    w = _small(N=777, C=16, K=4, causal=True, dtype="bf16")
    x = workloads.prefill_inputs(w)
    t = w.N - 1
    pyr = oracle.build_pyramid(x["k"], w.C)
    rows = [(0, h, t) for h in range(w.H_kv)]
    s1, _ = oracle.select_rows(_cfg(oracle, w), x["q"], x["k"], pyr, rows)
    s2, _ = oracle.select_rows(_cfg(oracle, w.with_(causal=False)), x["q"], x["k"], pyr, rows)
    assert (s1 == s2).all()
    # Held query rows can start anywhere (decode passes one row).
    q1 = x["q"][:, :, t:t + 1, :].contiguous()
    s3, _ = oracle.select_rows(_cfg(oracle, w, Nq=1, q_t0=t), q1, x["k"], pyr, rows)
    assert (s1 == s3).all()


@pytest.mark.parametrize("causal", [True, False])
def test_held_query_block_gives_the_whole_sequence_rows(oracle, causal):
    # A block of query rows held at an unaligned offset (a sequence-parallel
    # shard, or decode's single row) must give the rows that the whole
    # sequence's queries give: row j of the block is position q_t0 + j.
    w = _small(N=600, C=16, K=4, causal=causal, dtype="bf16", seed=91)
    x = workloads.prefill_inputs(w)
    pyr = oracle.build_pyramid(x["k"], w.C)
    a, b = 123, 411
    rng = np.random.default_rng(5)
    ts = np.unique(np.concatenate([[a, b - 1], rng.integers(a, b, 40)]))
    rows = [(0, h, int(t)) for h in range(w.H_kv) for t in ts]
    s_all, g_all = oracle.select_rows(_cfg(oracle, w), x["q"], x["k"], pyr, rows)
    qb = x["q"][:, :, a:b].contiguous()
    cfg_b = _cfg(oracle, w, Nq=b - a, q_t0=a)
    s_blk, g_blk = oracle.select_rows(cfg_b, qb, x["k"], pyr, rows)
    assert (s_all == s_blk).all() and np.array_equal(g_all, g_blk)
    o_all, l_all = oracle.attn_rows(_cfg(oracle, w), x["q"], x["k"], x["v"], rows, s_all)
    o_blk, l_blk = oracle.attn_rows(cfg_b, qb, x["k"], x["v"], rows, s_all)
    assert np.array_equal(o_all, o_blk) and np.array_equal(l_all, l_blk)
    if causal:
        # The offset matters under the causal reading: the block read as if
        # it started at position 0 sees fewer blocks and selects differently.
        s_wrong, _ = oracle.select_rows(_cfg(oracle, w, Nq=b - a, q_t0=0), qb, x["k"], pyr,
                                        [(0, h, int(t) - a) for h in range(w.H_kv) for t in ts])
        assert not (s_wrong == s_all).all()
