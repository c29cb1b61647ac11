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
