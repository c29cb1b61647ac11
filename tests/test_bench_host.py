"""Host-side measurement helpers of bench.py (no GPU): the recall of one
selection against another, the planted-needle recall, and the traffic
record's staleness check."""
import json
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_recall_at_k_counts_shared_valid_entries():
    sel = torch.tensor([[[[0, 3, 5, -1]], [[1, 2, 4, 7]]]], dtype=torch.int32)
    ref = torch.tensor([[[[0, 5, 6, -1]], [[1, 2, 3, 4]]]], dtype=torch.int32)
    # row 0: {0, 5} of {0, 5, 6}; row 1: {1, 2, 4} of {1, 2, 3, 4}
    assert bench.recall_at_k(sel, ref) == 5 / 7
    assert bench.recall_at_k(ref, ref) == 1.0
    # Chunking does not change the result.
    assert bench.recall_at_k(sel, ref, chunk=1) == 5 / 7


def test_needle_recall_over_rows_and_heads():
    sel = torch.full((1, 2, 10, 3), -1, dtype=torch.int32)
    sel[0, 0, 5] = torch.tensor([1, 2, 3])
    sel[0, 1, 5] = torch.tensor([0, 4, 6])
    sel[0, 0, 7] = torch.tensor([0, 1, 5])
    assert bench.needle_recall(sel, [(5, 2), (7, 5)]) == 0.5
    assert bench.needle_recall(sel, []) is None


def test_traffic_record_is_dropped_when_a_source_changes(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    import hashlib
    rec = {"w": {"attn": {"sources": ["k.cu"], "sha256": hashlib.sha256(b"kernel v1").hexdigest(),
                          "dram_read_bytes": 10, "dram_write_bytes": 5}}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("w", "attn") == 15
    src.write_text("kernel v2")
    assert bench.measured_traffic("w", "attn") is None
    assert bench.measured_traffic("other", "attn") is None


def test_cpu_decode_baseline_on_a_small_decode_workload():
    """The decode CPU baseline runs the oracle's append, selection and
    attention for a whole step's sequences when they fit the budget, and
    labels what it timed."""
    from hierarchical_top_block_mean_b200 import workloads
    wd = workloads.DECODE["decode_64x128k"].with_(name="dec_tiny", S=3, context=700, H_q=8, H_kv=2)
    r = bench.cpu_decode_baseline(wd, budget_s=1.0)
    assert r["kind"] == "oracle" and r["us_per_step"] > 0 and r["cores"] >= 1
    assert "3 steps" in r["sample"] and "701 tokens" in r["sample"]


def test_work_model_matches_the_oracle_trace(oracle):
    """The bench's algorithmic work model counts, per query row, the leaf
    candidates the search scores and the child summaries the router gathers
    from the level geometry alone. The oracle's per-level trace gives the true
    counts: the model may only over-count a block whose second child starts
    after t, so it stays within a few percent above the truth."""
    import numpy as np
    from hierarchical_top_block_mean_b200 import workloads
    w = workloads.Prefill("model", B=1, N=3000, H_q=4, H_kv=1, d=16, C=16, K=4, causal=True, dtype="f32", seed=3)
    x = workloads.prefill_inputs(w)
    cfg = oracle.make_cfg(B=1, N=w.N, H_q=w.H_q, H_kv=w.H_kv, d=w.d, C=w.C, K=w.K, causal=True, dtype_code=0)
    pyr = oracle.build_pyramid(x["k"], w.C)
    rows = np.array([(0, 0, t) for t in range(w.N)], np.int64)
    _, _, tr = oracle.select_rows(cfg, x["q"], x["k"], pyr, rows, trace=True)
    scored = tr["n"] > w.K
    pairs = int(np.where(scored[:, 1], tr["n"][:, 1], 0).sum())
    sizes, _ = oracle.geometry(w.N, w.C)
    gathered = 0
    for r, t in enumerate(range(w.N)):
        for l in range(2, len(sizes)):
            if scored[r, l]:
                for s in range(tr["n"][r, l]):
                    i = tr["cand"][r, l, s]
                    gathered += sum(1 for c in (2 * i, 2 * i + 1)
                                    if c < sizes[l - 1] and c * (w.C << (l - 2)) <= t)
    m = bench.work_model(w)
    assert pairs <= m["leaf_pairs"] <= 1.05 * pairs
    assert m["leaf_flops"] == m["leaf_pairs"] * 2 * (w.H_q // w.H_kv) * w.C * w.d
    assert gathered * w.d * 4 <= m["router_gather_bytes"] <= 1.10 * gathered * w.d * 4


def test_work_model_leaves_out_the_tensor_core_router_levels():
    """At G_Q = 8, d = 128 (bf16) the router reads the node scores of each
    16-query block's top three scored levels (taken at the block's last query)
    instead of gathering children. The work model must count gathers only on
    the other scored levels, and the tensor-core pass's children rows on
    those three. Checked against a per-position loop over the level geometry."""
    from hierarchical_top_block_mean_b200 import workloads
    w = workloads.Prefill("model_g8", B=1, N=5000, H_q=8, H_kv=1, d=128, C=64, K=16, causal=True, dtype="bf16",
                          seed=3)
    m = bench.work_model(w)
    L = 1
    while -(-w.N // (w.C << (L - 1))) > 1:
        L += 1
    size = {l: -(-w.N // (w.C << (l - 1))) for l in range(1, L + 1)}

    def valid(l, t):
        return min(size[l], t // (w.C << (l - 1)) + 1)

    def start(t):
        l = L
        while l >= 1 and valid(l, t) <= w.K:
            l -= 1
        return l

    gathered = 0
    for t in range(w.N):
        top = start(min(w.N - 1, (t // 16) * 16 + 15))
        started = False
        for l in range(L, 1, -1):
            v = valid(l, t)
            scored = started or v > w.K
            if scored and not (top - 2 <= l <= top):
                gathered += 2 * (min(2 * w.K, v) if started else v)
            started = scored
    rows = 0
    for blk in range(-(-w.N // 16)):
        last = min(w.N - 1, blk * 16 + 15)
        top = start(last)
        for i in range(3):
            l = top - i
            if l < 2:
                break
            rows += min(2 * valid(l, last), size[l - 1])
    assert m["router_gather_bytes"] == gathered * w.d * 4
    assert m["router_top_flops"] == rows * 2 * 2 * 128 * w.d
    # and with the tensor-core pass off (f32), every scored level is gathered
    m32 = bench.work_model(w.with_(dtype="f32"))
    assert m32["router_top_flops"] == 0 and m32["router_gather_bytes"] > m["router_gather_bytes"]


def test_clock_sampler_covers_a_short_timed_region(tmp_path, monkeypatch):
    """nvidia-smi takes a while to start; the sampler must wait for its first
    sample so that a timed region shorter than that still gets samples, and it
    must report only the samples taken during the region. A fake nvidia-smi on
    PATH (0.3 s start-up, a sample every 50 ms) stands in for the real one."""
    import os
    import time
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/sh\nsleep 0.3\nwhile true; do\n"
                    "  echo '0, 1965, 1965, 500.0, 0x4, Not Active, Not Active, Not Active, Active'\n"
                    "  sleep 0.05\ndone\n")
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ.get("PATH", ""))
    with bench.ClockSampler(0) as clk:
        time.sleep(0.2)  # the timed region
    s = clk.summary()
    assert s["sampled"] == "during the timed region"
    assert s["samples"] >= 1
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
