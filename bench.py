#!/usr/bin/env python
"""Benchmark of the PISA prefill hot path on B200.

One step = mean-pooled key pyramid + PISA top-K selection + block-sparse
attention over one full synthetic input (default: 262144 tokens, 16 query
heads, 2 kv heads, d = 128, C = 64, K = 16, bf16, causal, 256 planted
needles). The flat single-level selector and the decode step (64 sequences x
131072 cached tokens) are timed beside it and reported in the same line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--seq-parallel]

Under torchrun each rank runs the same workload on its own GPU (weak
scaling: the path shards over independent sequences and heads with no
collective); the barrier-bracketed time is the max over ranks. With
--seq-parallel the ranks instead split one sequence by position and
all-gather its keys and values over NCCL (strong scaling).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import tempfile
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hierarchical_top_block_mean_b200 import api, seqpar, workloads  # noqa: E402

METRIC = "PISA prefill tokens/s (select+attn) at 64K/256K; decode select µs/step"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers

def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return FALLBACK_PEAKS, "fallback"


def dist_init(n_gpus):
    if n_gpus > 1 or "RANK" in os.environ:
        import torch.distributed as dist
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
        return dist
    return None


def aggregate(dist, local_ms: float, local_tokens: int):
    """Whole-job result of one timed region: the max over ranks of the
    device time, and the tokens all ranks processed in it."""
    ms = max_over_ranks(dist, local_ms)
    world = dist.get_world_size() if dist else 1
    return ms, local_tokens * world / (ms * 1e-3)


def max_over_ranks(dist, x: float) -> float:
    if dist is None:
        return x
    dev = torch.device("cuda") if torch.cuda.is_available() else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"pisa_bench_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return self
        # nvidia-smi takes a few hundred ms to start; a timed region of a few
        # hundred ms would otherwise end before its first sample. Wait (up to
        # 5 s) for the first sample, and count the samples taken before the
        # region so that the summary can leave them out.
        t_end = time.time() + 5.0
        while time.time() < t_end and self.proc.poll() is None and self._lines() == 0:
            time.sleep(0.02)
        self.before = self._lines()
        return self

    def _lines(self):
        try:
            with open(self.path) as f:
                return sum(1 for line in f if line.strip())
        except OSError:
            return 0

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            lines = [line for line in f if line.strip()]
        # Samples taken during the region; the last one taken just before it
        # stands in only when the region was shorter than the sampling period.
        during = lines[getattr(self, "before", 0):]
        for line in (during if during else lines[-1:]):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "sampled": "during the timed region" if during else "just before the timed region"}


def events(n):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


# -------------------------------------------------------------- algorithmic models

def attn_bytes(w) -> float:
    """Bytes the sparse attention must move per launch: q and out once, plus
    the K and V rows of each row's selected blocks (per kv head and query:
    K blocks of C keys, causally clipped), with no reuse across queries."""
    e = 2 if w.dtype == "bf16" else 4
    qo = 2 * w.B * w.H_q * w.N * w.d * e
    keys = 0
    for t in range(0, w.N, max(1, w.N // 4096)):
        keys += min(w.K * w.C, t + 1)
    keys *= w.N / len(range(0, w.N, max(1, w.N // 4096)))
    return qo + 2 * w.B * w.H_kv * keys * w.d * e


def _valid(w, l, t):
    """Blocks of level l usable by queries at positions t (numpy array)."""
    import numpy as np
    M = -(-w.N // (w.C << (l - 1)))
    if not w.causal:
        return np.full(t.shape, M, dtype=np.int64)
    return np.minimum(M, t // (w.C << (l - 1)) + 1)


def work_model(w):
    """Algorithmic work per launch of each prefill kernel, from the level
    geometry alone (one pass over every query position t):
      router: per query row and scored inner level l >= 2, up to 2K
        candidates, each gathering its <= 2 child summaries (d fp32 values,
        stored as bf16 hi + lo) from L2, except on the levels the tensor-core
        pass scores (router_top_flops: 2 x 2 x 128 x d per child row of a
        16-query block's top three levels, hi and lo);
      leaf scorer: (query, candidate leaf) pairs at the leaf level, each
        2 G_Q C d flops;
      attention: 4 G_Q d flops per usable key of the K selected blocks;
      flat selector: 2 d flops per (query row, usable leaf) after the group sum;
      exact selector: 2 G_Q C d flops per (query row, usable leaf)."""
    import numpy as np
    t = np.arange(w.N, dtype=np.int64)
    L = api.pyramid_geometry(w.N, w.C)[0]
    K, G, e = w.K, w.H_q // w.H_kv, (2 if w.dtype == "bf16" else 4)
    heads = w.B * w.H_kv
    # Levels scored on tensor cores for G_Q = 8, d = 128 (bf16, K <= 16, C =
    # 64): the top three scored levels of each block of 16 queries,
    # taken at the block's last query; those levels are read, not gathered.
    dense = (w.dtype == "bf16" and w.d == 128 and G == 8 and K <= 16 and w.C == 64)
    last = np.minimum(w.N - 1, (t // 16) * 16 + 15)
    ltop = np.zeros(w.N, dtype=np.int64)
    for l in range(L, 0, -1):
        ltop = np.where((ltop == 0) & (_valid(w, l, last) > K), l, ltop)
    gathered = np.zeros(w.N)
    started = np.zeros(w.N, dtype=bool)
    for l in range(L, 1, -1):
        v = _valid(w, l, t)
        scored = started | (v > K)
        cand = np.where(started, np.minimum(2 * K, v), v)
        in_dense = dense & (l <= ltop) & (l >= ltop - 2)
        gathered += np.where(scored & ~in_dense, cand * 2, 0)
        started = scored
    # Children rows the tensor-core levels multiply per block (hi and lo parts).
    top_rows = 0.0
    if dense:
        blocks_last = last[::16]
        for i in range(3):
            lb = ltop[::16] - i
            ok = lb >= 2
            for l in np.unique(lb[ok]):
                sel = ok & (lb == l)
                size_below = -(-w.N // (w.C << (int(l) - 2)))
                top_rows += np.minimum(2 * _valid(w, int(l), blocks_last[sel]), size_below).sum()
    v1 = _valid(w, 1, t)
    pairs = np.where(v1 > K, np.where(started, np.minimum(2 * K, v1), v1), 0)
    keys = np.minimum(K * w.C, t + 1) if w.causal else np.full(w.N, min(K * w.C, w.N))
    return {k: float(v) for k, v in {
        "router_gather_bytes": heads * gathered.sum() * w.d * 4,
        "router_hbm_bytes": w.B * w.H_q * w.N * w.d * e + heads * w.N * (32 + 1) * 4,
        "leaf_pairs": heads * pairs.sum(),
        "leaf_flops": heads * pairs.sum() * 2 * G * w.C * w.d,
        "attn_flops": heads * keys.sum() * 4 * G * w.d,
        "attn_unique_bytes": (2 * w.B * w.H_q * w.N * w.d * e + 2 * heads * w.N * w.d * e + w.B * w.H_q * w.N * 4),
        "flat_flops": heads * v1.sum() * 2 * w.d,
        "exact_flops": heads * v1.sum() * 2 * G * w.C * w.d,
        "final_bytes": heads * w.N * (32 * 8 + K * 4),
        "attn_partial_bytes": heads * w.N * K * G * (128 * 2 + 8),
        "attn_out_bytes": w.B * w.H_q * w.N * (w.d * e + 4),
        "split_bytes": heads * api.pyramid_rows(w.N, w.C) * w.d * 8,
        "router_top_flops": heads * top_rows * 2 * 2 * 128 * w.d,
    }.items()}


def decode_bytes(wd) -> float:
    """HBM bytes one decode step must read, per (sequence, kv head): the
    group's queries, the child summaries of up to 2K candidates per scored
    inner level (fp32), the raw keys of up to 2K candidate leaves, and the
    values of the K selected leaves; plus the append's leaf and ancestor
    rows. Taken at the workload's starting length."""
    n = wd.context + 1
    L = api.pyramid_geometry(n, wd.C)[0]
    scored_inner = sum(1 for l in range(2, L + 1) if -(-n // (wd.C << (l - 2))) > wd.K)
    per = (wd.G_Q * wd.d * 2 + scored_inner * 2 * wd.K * 2 * wd.d * 4 + 2 * wd.K * wd.C * wd.d * 2
           + wd.K * wd.C * wd.d * 2 + L * 3 * wd.d * 4 + 2 * wd.d * 2)
    return wd.S * wd.H_kv * per


def pyramid_bytes(w) -> float:
    e = 2 if w.dtype == "bf16" else 4
    R = api.pyramid_rows(w.N, w.C)
    return w.B * w.H_kv * (w.N * w.d * e + R * w.d * 4)


def recall_at_k(sel, ref, chunk=1 << 16):
    """Mean over rows of |sel_row & ref_row| / |ref_row| for [..., K] index
    tensors padded with -1 (computed on the device in row chunks)."""
    a = sel.reshape(-1, sel.shape[-1])
    b = ref.reshape(-1, ref.shape[-1])
    hit = 0
    tot = 0
    for i in range(0, a.shape[0], chunk):
        x, y = a[i:i + chunk], b[i:i + chunk]
        eq = (x[:, :, None] == y[:, None, :]) & (y[:, None, :] >= 0)
        hit += int(eq.any(1).sum().item())
        tot += int((y >= 0).sum().item())
    return hit / max(tot, 1)


def needle_recall(sel, needles):
    """Share of planted (query position t, leaf j) needles, over every batch
    row and kv head, whose leaf j is among the K selected for t."""
    if not needles:
        return None
    ts = torch.tensor([t for t, _ in needles], device=sel.device)
    js = torch.tensor([j for _, j in needles], device=sel.device, dtype=sel.dtype)
    got = sel[:, :, ts, :]  # [B, H_kv, n, K]
    return float((got == js[None, None, :, None]).any(-1).float().mean().item())


def measured_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of `kernel` recorded by an ncu capture in
    profiles/traffic.json, or None when absent or when any of the kernel's
    source files has changed since the capture (the recorded sha256 of the
    concatenated sources no longer matches)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[workload][kernel]
        h = hashlib.sha256()
        for src in rec["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["sha256"]:
            return None
        return rec["dram_read_bytes"] + rec["dram_write_bytes"]
    except (OSError, KeyError, ValueError):
        return None


def kernel_rooflines(w, kern, flat_ms, exact_ms, decode, pk, pk_kind):
    """Each kernel's achieved rate against its binding roof: algorithmic work
    per launch (work_model, pyramid_bytes, decode_bytes) over the kernel's
    CUDA-event time per launch. Tensor-bound kernels use the measured bf16
    dense peak (burst: each is a single launch of at most a few tens of ms);
    memory-bound ones the measured HBM copy peak."""
    m = work_model(w)
    hbm, tf = pk["hbm_gbs"], pk["bf16_tflops"]
    out = {}

    def add(name, ms, launches, bound, work, note, **extra):
        if ms is None or ms <= 0:
            return
        if bound == "tensor":
            ach, peak, unit = work / (ms * 1e-3) / 1e12, tf, "TFLOP/s"
        else:
            ach, peak, unit = work / (ms * 1e-3) / 1e9, hbm, "GB/s"
        out[name] = dict(ms=ms, launches=launches, bound=bound, achieved=ach, peak=peak, unit=unit,
                         frac=ach / peak, peak_kind=pk_kind, work=work,
                         work_unit="flop" if bound == "tensor" else "byte", note=note, **extra)

    def k(name):
        return kern.get(name, (None, 0))

    add("pyramid_kernel", *k("pyramid_kernel"), "hbm", pyramid_bytes(w),
        "keys read once + fp32 pyramid written once (one cooperative launch)")
    add("split_kernel", *k("split_kernel"), "hbm", m["split_bytes"], "fp32 pyramid read, bf16 hi/lo planes written")
    add("router_top_kernel", *k("router_top_kernel"), "tensor", m["router_top_flops"],
        "hi and lo products of 128 (query, head) rows with the children of the top three scored levels of each "
        "16-query block")
    r = k("router_kernel")
    if r[0]:
        add("router_kernel", *r, "hbm", m["router_hbm_bytes"],
            "HBM bytes: queries + candidate lists; its real limit is the L2 gather of child summaries",
            l2_gather_gbs=m["router_gather_bytes"] / (r[0] * 1e-3) / 1e9, l2_gather_bytes=m["router_gather_bytes"])
    for leaf in ("leaf_umma_kernel", "leaf_kernel"):
        add(leaf, *k(leaf), "tensor", m["leaf_flops"], f"{m['leaf_pairs']:.4g} (query, leaf) pairs x 2 G_Q C d")
    add("final_kernel", *k("final_kernel"), "hbm", m["final_bytes"], "2K (score, leaf) pairs read + K written per row")
    a = k("attn_kernel")
    if a[0]:
        add("attn_kernel", *a, "tensor", m["attn_flops"], "4 G_Q d flops per usable key of the K selected blocks",
            hbm_unique_gbs=m["attn_unique_bytes"] / (a[0] * 1e-3) / 1e9,
            hbm_unique_frac=m["attn_unique_bytes"] / (a[0] * 1e-3) / 1e9 / hbm,
            l2_gather_gbs=attn_bytes(w) / (a[0] * 1e-3) / 1e9)
    ab = k("attn_bucket_kernel")
    if ab[0]:
        add("attn_bucket_kernel", *ab, "tensor", m["attn_flops"],
            "4 G_Q d flops per usable key of the K selected blocks; also writes the partial states",
            partial_write_gbs=m["attn_partial_bytes"] / (ab[0] * 1e-3) / 1e9)
    add("attn_merge_kernel", *k("attn_merge_kernel"), "hbm", m["attn_partial_bytes"] + m["attn_out_bytes"],
        "partial states of every (query, selected block, head) read once; out and lse written")
    add("flat_selector", flat_ms, 1, "tensor", m["flat_flops"],
        "one pisa_select_flat call (flat_prep_kernel + flat_umma_kernel at d = 128); 2 d flops per "
        "(query row, usable leaf) after the group sum; not part of the step")
    add("exact_umma_kernel", exact_ms, 1, "tensor", m["exact_flops"],
        "2 G_Q C d flops per (query row, usable leaf); not part of the step")
    if decode:
        wd = workloads.DECODE[decode["workload"]]
        add("decode_kernel", decode["us_per_step"] * 1e-3, 1, "hbm", decode_bytes(wd),
            "fused step: summaries of scored levels, candidate leaf keys, selected values, append rows")
    return out


# ------------------------------------------------------------------ arms

def cpu_baseline(w, x, budget_s=15.0):
    """The fp64 CPU oracle as it stands, on a bounded sample: the full
    pyramid plus select + attention for a seeded sample of rows, scaled to
    tokens/s over all rows."""
    import numpy as np
    import oracle as O
    O.build()
    cores = len(os.sched_getaffinity(0))
    qh, kh, vh = (x[n].detach().cpu().contiguous() for n in ("q", "k", "v"))
    cfg = O.make_cfg(B=w.B, N=w.N, H_q=w.H_q, H_kv=w.H_kv, d=w.d, C=w.C, K=w.K, causal=w.causal,
                     dtype_code=0 if w.dtype == "f32" else 1)
    t0 = time.perf_counter()
    pyr = O.build_pyramid(kh, w.C)
    t_pyr = time.perf_counter() - t0
    rng = np.random.default_rng(0)
    n_rows, t_rows = 0, 0.0
    batch = 64
    while t_rows < budget_s and n_rows < w.B * w.H_kv * w.N:
        ts = rng.integers(0, w.N, batch)
        hs = rng.integers(0, w.H_kv, batch)
        rows = np.stack([np.zeros(batch, np.int64), hs, ts], 1)
        t1 = time.perf_counter()
        sel, _ = O.select_rows(cfg, qh, kh, pyr, rows)
        O.attn_rows(cfg, qh, kh, vh, rows, sel)
        t_rows += time.perf_counter() - t1
        n_rows += batch
    total_rows = w.B * w.H_kv * w.N
    est = t_pyr + t_rows * total_rows / n_rows
    return {"value": w.B * w.N / est, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 oracle: full pyramid ({t_pyr:.1f} s) + select+attention on {n_rows} random "
                      f"(kv head, query) rows ({t_rows:.1f} s), extrapolated linearly to all {total_rows} rows"}


def cpu_decode_baseline(wd, budget_s=5.0):
    """The fp64 CPU oracle as it stands, on a bounded sample of the decode
    step. The sample is one sequence at the workload's context length with
    all its kv heads, timed per step for the append's pyramid update (per
    head), the root-to-leaf selection and the attention of the new token (all
    heads' rows in one call each, which the oracle spreads over its threads).
    The prefix pyramid is the cached state and is built untimed. The result
    is scaled linearly to all S sequences."""
    import numpy as np
    import oracle as O
    O.build()
    cores = len(os.sched_getaffinity(0))
    n = wd.context + 1  # tokens held once the step's token is appended
    cfg = O.make_cfg(B=1, N=n, H_q=wd.H_q, H_kv=wd.H_kv, d=wd.d, C=wd.C, K=wd.K, causal=True, dtype_code=1,
                     Nq=1, q_t0=n - 1)
    _, offs_c = O.geometry(wd.cap, wd.C)
    g = torch.Generator().manual_seed(wd.seed + 77)
    # One sequence's cache serves every timed step: the work does not depend
    # on the cached values, and each step draws its own query.
    k = torch.randn(1, wd.H_kv, n, wd.d, generator=g).to(torch.bfloat16)
    v = torch.randn(1, wd.H_kv, n, wd.d, generator=g).to(torch.bfloat16)
    pyr = O.build_pyramid(k, wd.C)
    cap_pyr = [np.zeros((offs_c[-1], wd.d), np.float64) for _ in range(wd.H_kv)]
    rows = [(0, h, n - 1) for h in range(wd.H_kv)]
    t_step, seqs = 0.0, 0
    while seqs < wd.S and (seqs == 0 or t_step < budget_s):
        q = torch.randn(1, wd.H_q, 1, wd.d, generator=g).to(torch.bfloat16)
        t0 = time.perf_counter()
        for h in range(wd.H_kv):
            O.decode_append(k[0, h], n - 1, wd.C, wd.cap, cap_pyr[h])
        sel, _ = O.select_rows(cfg, q, k, pyr, rows)
        O.attn_rows(cfg, q, k, v, rows, sel)
        t_step += time.perf_counter() - t0
        seqs += 1
    us = t_step / seqs * wd.S * 1e6
    return {"us_per_step": us, "cores": cores, "kind": "oracle",
            "sample": f"fp64 oracle: append + select + attention of the new token for {seqs} steps of one "
                      f"sequence ({wd.H_kv} kv heads) at {n} tokens ({t_step:.2f} s), extrapolated linearly "
                      f"to {wd.S} sequences; {wd.H_kv} rows per oracle call"}


def run_reference(args):
    """Reference arm: the CPU oracle as it stands, timed on the host cores.
    Under torchrun only rank 0 runs it; the other ranks exit without work
    (there is nothing to exchange, so no process group is created)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = workloads.PREFILL[args.workload]
    x = workloads.prefill_inputs(w, device="cpu")
    budget = args.ref_step_budget or max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(w, x, budget_s=budget)
    vals = [cpu_baseline(w, x, budget_s=budget) for _ in range(args.steps)]
    v = statistics.median(r["value"] for r in vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": w.B * w.N / v * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "N": w.N, "H_q": w.H_q, "H_kv": w.H_kv, "d": w.d, "C": w.C,
                       "g": 2, "K": w.K, "q_tile": 4, "causal": w.causal, "structure": w.structure,
                       "input_dtype": w.dtype},
            "ms_per_step_kind": "extrapolated: each step times the full pyramid plus a random row sample and "
                                "scales the row time linearly to all rows",
            "cpu_baseline": dict(vals[-1], value=v),
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def _reset_decode(st, lens0):
    """Back to the cached context: lengths restored, pyramids rebuilt."""
    st.len.copy_(lens0)
    st.init()


def time_decode(wd, warmup=4):
    """µs per decode step over the workload's full run of wd.steps steps
    (context -> context + steps tokens per sequence): append + fused select
    + attention per step. Then, from the same starting state, the selection
    alone, the attention alone and the append alone, each over wd.steps
    launches. Warm-up steps run first and the state is reset after them."""
    dev = torch.device("cuda")
    steps = wd.steps
    kc, vc, lens = workloads.decode_cache(wd, device=dev)
    lens0 = lens.clone()
    st = api.DecodeState(S=wd.S, cap=wd.cap, H_q=wd.H_q, H_kv=wd.H_kv, d=wd.d, C=wd.C, K=wd.K,
                         dtype=wd.torch_dtype, device=dev, k_cache=kc, v_cache=vc, lens=lens)
    st.init()
    ins = [workloads.decode_step_inputs(wd, s, device=dev) for s in range(steps)]
    for s in range(warmup):
        st.step(*ins[s], keep_sel=False)
    _reset_decode(st, lens0)
    e0, e1 = events(2)
    torch.cuda.synchronize()
    e0.record()
    for s in range(steps):
        st.step(*ins[s], keep_sel=False)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / steps
    ok = int(st.status.item()) == 0
    end_len = int(st.len.min().item())
    _reset_decode(st, lens0)
    q = ins[0][0]
    st.select(q)
    torch.cuda.synchronize()
    e0.record()
    for s in range(steps):
        st.select(ins[s][0])
    e1.record()
    torch.cuda.synchronize()
    us_sel = e0.elapsed_time(e1) * 1e3 / steps
    # Attention alone over the selection just made, then the append alone
    # (each its own launch; the append advances every sequence by one token).
    e0.record()
    for s in range(steps):
        st.attend(ins[s][0])
    e1.record()
    torch.cuda.synchronize()
    us_attn = e0.elapsed_time(e1) * 1e3 / steps
    e0.record()
    for s in range(steps):
        st.append(ins[s][1], ins[s][2])
    e1.record()
    torch.cuda.synchronize()
    us_app = e0.elapsed_time(e1) * 1e3 / steps
    ok = ok and int(st.status.item()) == 0
    del st, kc, vc
    torch.cuda.empty_cache()
    return {"workload": wd.name, "us_per_step": us, "select_us": us_sel, "attn_us": us_attn, "append_us": us_app,
            "steps": steps, "tokens": [wd.context, end_len], "status_ok": ok}


def time_decode_paged(wd, warmup=4):
    """µs per fused decode step over paged caches: the same workload and
    number of steps with each sequence's leaf blocks in pages of a shuffled
    pool (one leaf per page)."""
    dev = torch.device("cuda")
    steps = wd.steps
    kc, vc, lens = workloads.decode_cache(wd, device=dev)
    max_pages = wd.cap // wd.C
    perm = torch.randperm(wd.S * max_pages, generator=torch.Generator().manual_seed(1)).to(dev)

    def pages(x):
        y = x.reshape(wd.S, wd.H_kv, max_pages, wd.C, wd.d).permute(0, 2, 1, 3, 4).reshape(-1, wd.H_kv, wd.C, wd.d)
        out = torch.empty_like(y)
        out[perm] = y  # logical page i of the pool goes to physical page perm[i]
        return out

    kp = pages(kc)
    del kc
    vp = pages(vc)
    del vc
    bt = perm.reshape(wd.S, max_pages).to(torch.int32).contiguous()
    lens0 = lens.clone()
    st = api.PagedDecodeState(S=wd.S, max_pages=max_pages, H_q=wd.H_q, H_kv=wd.H_kv, d=wd.d, C=wd.C, K=wd.K,
                              k_pages=kp, v_pages=vp, block_table=bt, lens=lens, dtype=wd.torch_dtype)
    st.init()
    ins = [workloads.decode_step_inputs(wd, s, device=dev) for s in range(steps)]
    for s in range(warmup):
        st.step(*ins[s], keep_sel=False)
    _reset_decode(st, lens0)
    e0, e1 = events(2)
    torch.cuda.synchronize()
    e0.record()
    for s in range(steps):
        st.step(*ins[s], keep_sel=False)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / steps
    ok = int(st.status.item()) == 0
    del st, kp, vp
    torch.cuda.empty_cache()
    return {"workload": wd.name + " (paged)", "us_per_step": us, "steps": steps, "status_ok": ok}


def run_gpu(args):
    dist = dist_init(args.gpus)
    rank = dist.get_rank() if dist else 0
    world = dist.get_world_size() if dist else 1
    dev = torch.device("cuda", torch.cuda.current_device())
    w = workloads.PREFILL[args.workload]
    x = workloads.prefill_inputs(w, device=dev)
    q, k, v = x["q"], x["k"], x["v"]
    pr = api.Problem.of(q, k, C=w.C, K=w.K, causal=w.causal)
    p = api.Prefill(pr, dev)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        p(q, k, v)
    torch.cuda.synchronize()

    n_ev = 4
    evs = [events(n_ev) for _ in range(args.steps)]
    launches0 = api.launch_count()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0 = time.perf_counter()
        for s in range(args.steps):
            e = evs[s]
            e[0].record(stream)
            p.pyramid(k)
            e[1].record(stream)
            p.select(q, k)
            e[2].record(stream)
            p.attend(q, k, v)
            e[3].record(stream)
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
        if dist:
            dist.barrier()
    launches = api.launch_count() - launches0
    stage = {"pyramid": 0.0, "select": 0.0, "attn": 0.0}
    for e in evs:
        stage["pyramid"] += e[0].elapsed_time(e[1])
        stage["select"] += e[1].elapsed_time(e[2])
        stage["attn"] += e[2].elapsed_time(e[3])
    dev_ms = sum(e[0].elapsed_time(e[3]) for e in evs) / args.steps
    ms, value = aggregate(dist, dev_ms, w.B * w.N)
    stage_ms = {kk: vv / args.steps for kk, vv in stage.items()}

    # Per-kernel device time: the same steps again, outside the timed region,
    # with every library launch bracketed by CUDA events on its stream.
    with api.KernelTimer() as kt:
        for _ in range(args.steps):
            p(q, k, v)
    kern_ms = {n: (t_ms / args.steps, c / args.steps) for n, (t_ms, c) in kt.result.items()}

    # Exact-score flat selector (every usable leaf scored by its raw-key LSE)
    # on the same inputs, once after a warm-up, and the share of its top-K
    # leaves that the pyramid search keeps.
    pisa_sel = p.sel.clone()
    xsel = api.select_exact(q, k, C=w.C, K=w.K, causal=w.causal)
    xe0, xe1 = events(2)
    xe0.record(stream)
    api.select_exact(q, k, C=w.C, K=w.K, causal=w.causal, out=xsel)
    xe1.record(stream)
    torch.cuda.synchronize()
    exact_ms = xe0.elapsed_time(xe1)
    recall = recall_at_k(pisa_sel, xsel)
    needles = ({"pisa": needle_recall(pisa_sel, x["needles"]), "exact": needle_recall(xsel, x["needles"])}
               if x["needles"] else None)
    del pisa_sel, xsel

    # Flat single-level selector on the same inputs (its own launches).
    fe0, fe1 = events(2)
    api.select_flat(q, p.pyr, C=w.C, K=w.K, causal=w.causal, H_kv=w.H_kv)
    fe0.record(stream)
    for _ in range(args.steps):
        api.select_flat(q, p.pyr, C=w.C, K=w.K, causal=w.causal, H_kv=w.H_kv, out=p.sel)
    fe1.record(stream)
    torch.cuda.synchronize()
    flat_ms = fe0.elapsed_time(fe1) / args.steps
    if needles:
        needles["flat"] = needle_recall(p.sel, x["needles"])

    # Sequence-parallel split of the step over 8 GPUs, each GPU's share
    # timed here one after another on this GPU: the pyramid over all keys,
    # then the selection and attention of its eighth of the query rows. The
    # key and value all-gather that precedes them is not in these figures.
    seq_par = None
    if w.N % 8 == 0:
        shard_ms = []
        for r in range(8):
            a, n = seqpar.shard_span(w.N, 8, r)
            qs = q[:, :, a:a + n].contiguous()
            sh = api.PrefillShard(pr, a, n, dev)
            sh(qs, k, v)
            se0, se1 = events(2)
            se0.record(stream)
            sh(qs, k, v)
            se1.record(stream)
            torch.cuda.synchronize()
            shard_ms.append(se0.elapsed_time(se1))
            del qs, sh
        seq_par = {"shards": 8, "shard_ms": shard_ms, "max_shard_ms": max(shard_ms),
                   "balance": max(shard_ms) / (sum(shard_ms) / len(shard_ms)),
                   "note": "per-GPU compute of an 8-way sequence-parallel step (pyramid over all keys + "
                           "selection and attention of 1/8 of the queries), each shard timed once on this "
                           "GPU after a warm-up; the NVLink all-gather of K and V is not included"}

    # Attention backward over the step's selection (training), once after a
    # warm-up: dq, dk, dv (fp32) for a random output gradient.
    bwd_ms = None
    if w.dtype == "bf16":
        p(q, k, v)
        dout = torch.randn(q.shape, generator=torch.Generator(device=dev).manual_seed(11), device=dev).to(q.dtype)
        api.sparse_attn_bwd(q, k, v, p.sel, p.out, p.lse, dout, C=w.C, causal=w.causal)
        be0, be1 = events(2)
        be0.record(stream)
        grads = api.sparse_attn_bwd(q, k, v, p.sel, p.out, p.lse, dout, C=w.C, causal=w.causal)
        be1.record(stream)
        torch.cuda.synchronize()
        bwd_ms = be0.elapsed_time(be1)
        del grads, dout

    # End to end through the public API from pinned host buffers: every step
    # copies q, k, v in and the output back. PrefillStream overlaps step s's
    # compute with step s + 1's upload and step s - 1's download; the serial
    # form (copy in, compute, copy out, one after another) is reported beside it.
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hout = torch.empty(p.out.shape, dtype=p.out.dtype).pin_memory()
    e2e_steps = max(3, args.steps)  # pipeline fill and drain are inside the timed region
    ps = api.PrefillStream(pr, dev)
    ps.submit(hq, hk, hv, hout)  # warm-up
    ps.synchronize()
    torch.cuda.synchronize()
    ee0, ee1 = events(2)
    ee0.record(stream)
    ps.h2d.wait_stream(stream)
    for _ in range(e2e_steps):
        ps.submit(hq, hk, hv, hout)
    stream.wait_stream(ps.d2h)
    ee1.record(stream)
    torch.cuda.synchronize()
    e2e_ms, e2e_value = aggregate(dist, ee0.elapsed_time(ee1) / e2e_steps, w.B * w.N)
    del ps
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    torch.cuda.synchronize()
    se0, se1 = events(2)
    se0.record(stream)
    for _ in range(e2e_steps):
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        p(dq, dk, dv)
        hout.copy_(p.out, non_blocking=True)
    se1.record(stream)
    torch.cuda.synchronize()
    _, e2e_serial = aggregate(dist, se0.elapsed_time(se1) / e2e_steps, w.B * w.N)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = hout.numel() * hout.element_size()
    del hq, hk, hv, hout, dq, dk, dv

    decode = None
    if not args.no_decode:
        del x
        torch.cuda.empty_cache()
        decode = time_decode(workloads.DECODE[args.decode_workload])
        decode["paged"] = time_decode_paged(workloads.DECODE[args.decode_workload])
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            decode["cpu_baseline"] = cpu_decode_baseline(workloads.DECODE[args.decode_workload])

    pk, pk_kind = peaks()
    kernels = kernel_rooflines(w, kern_ms, flat_ms, exact_ms, decode, pk, pk_kind)
    # Measured DRAM bytes per launch (ncu capture in profiles/traffic.json, while the kernel's
    # sources are unchanged) over this run's time per launch: the kernel's DRAM rate.
    for name, kr in kernels.items():
        t = measured_traffic(w.name, name)
        if t is not None and kr.get("ms"):
            kr["traffic"] = t
            kr["dram_gbs"] = t / (kr["ms"] * 1e-3) / 1e9
            kr["dram_frac"] = kr["dram_gbs"] / pk["hbm_gbs"]
    # Roofline of the dominant kernel of the step (largest share of its time).
    step_kernels = [n for n in kern_ms if n in kernels]
    top = max(step_kernels, key=lambda n: kernels[n]["ms"])
    kr = kernels[top]
    roof = {"kernel": top, "bound": kr["bound"], "achieved": kr["achieved"], "peak": kr["peak"], "unit": kr["unit"],
            "frac": kr["frac"], "peak_kind": pk_kind, "share_of_step": kr["ms"] / ms,
            "traffic": measured_traffic(w.name, top), "work_per_launch": kr["work"], "work_unit": kr["work_unit"],
            "note": kr["note"]}
    for extra in ("hbm_unique_frac", "l2_gather_gbs"):
        if extra in kr:
            roof[extra] = kr[extra]

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "N": w.N, "H_q": w.H_q, "H_kv": w.H_kv, "d": w.d, "C": w.C,
                   "g": 2, "K": w.K, "q_tile": 4, "causal": w.causal, "structure": w.structure,
                   "l2": "inputs larger than L2 (q alone is %.0f MB)" % (q.numel() * q.element_size() / 1e6)},
        "stages_ms": stage_ms, "kernels": kernels, "flat_select_ms": flat_ms,
        "select_speedup_vs_flat": flat_ms / stage_ms["select"] if stage_ms["select"] > 0 else None,
        "exact_select_ms": exact_ms,
        "select_speedup_vs_exact": exact_ms / stage_ms["select"] if stage_ms["select"] > 0 else None,
        "pisa_recall_vs_exact": recall,
        "needle_recall": needles,
        "attn_bwd_ms": bwd_ms,
        "seq_parallel": seq_par,
        "decode": decode,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "overlap": "api.PrefillStream: step s+1's upload and step s-1's download overlap step s "
                           "(two copy streams, double-buffered slots)",
                "serial_value": e2e_serial},
        "gpu_launches": launches, "roofline": roof, "clocks": clk.summary(), "wall_s": wall,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        xh = workloads.prefill_inputs(w, device=dev)
        line["cpu_baseline"] = cpu_baseline(w, xh, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(line))
    if dist:
        dist.destroy_process_group()
    return 0


def run_seq_parallel(args):
    """One sequence split by position over the ranks (strong scaling): per
    step, the NCCL all-gather of the key and value slices, the pyramid, and
    the selection and attention of each rank's query rows
    (seqpar.SeqParallelPrefill). Without torchrun it runs one rank."""
    import datetime

    import torch.distributed as tdist
    dist = dist_init(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    if dist is None:
        tdist.init_process_group("nccl", store=tdist.HashStore(), rank=0, world_size=1, device_id=dev,
                                 timeout=datetime.timedelta(seconds=300))
        dist = tdist
    rank, world = dist.get_rank(), dist.get_world_size()
    w = workloads.PREFILL[args.workload]
    x = workloads.prefill_inputs(w, device=dev)  # the same seeded sequence on every rank
    q0, n = seqpar.shard_span(w.N, world, rank)
    q, k, v = (x[t][:, :, q0:q0 + n].contiguous() for t in ("q", "k", "v"))
    pr = api.Problem.of(x["q"], x["k"], C=w.C, K=w.K, causal=w.causal)
    del x
    torch.cuda.empty_cache()
    sp = seqpar.SeqParallelPrefill(pr, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        sp(q, k, v)
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    launches0 = api.launch_count()
    e0, e1 = events(2)
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            sp(q, k, v)
        e1.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
    launches = api.launch_count() - launches0
    ms = max_over_ranks(dist, e0.elapsed_time(e1) / args.steps)
    value = w.B * w.N / (ms * 1e-3)  # the whole sequence's tokens per step

    # End to end: this rank's slices from pinned host memory, its output rows back.
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hout = torch.empty(sp.shard.out.shape, dtype=sp.shard.out.dtype).pin_memory()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    e2e_steps = max(1, min(args.steps, 5))
    torch.cuda.synchronize()
    dist.barrier()
    ee0, ee1 = events(2)
    ee0.record(stream)
    for _ in range(e2e_steps):
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        sp(dq, dk, dv)
        hout.copy_(sp.shard.out, non_blocking=True)
    ee1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(dist, ee0.elapsed_time(ee1) / e2e_steps)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = hout.numel() * hout.element_size()
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "N": w.N, "H_q": w.H_q, "H_kv": w.H_kv, "d": w.d, "C": w.C,
                   "g": 2, "K": w.K, "q_tile": 4, "causal": w.causal, "parallelism": f"sp{world}",
                   "tokens_per_rank": n, "l2": "inputs larger than L2"},
        "e2e": {"value": w.B * w.N / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "per": "rank"},
        "gpu_launches": launches, "roofline": None, "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line))
    del sp
    dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="needle_256k", choices=sorted(workloads.PREFILL))
    ap.add_argument("--decode-workload", default="decode_64x128k", choices=sorted(workloads.DECODE))
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--seq-parallel", action="store_true",
                    help="split one sequence over the ranks by position (strong scaling) instead of a full "
                         "sequence per rank")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-step-budget", type=float, default=None,
                    help="seconds of oracle row work per step of the reference arm")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    if args.seq_parallel:
        return run_seq_parallel(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
