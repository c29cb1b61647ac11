"""Seeded synthetic inputs for the PISA hot path.

This module is shared by the tests, the benchmark and the smoke check. It only
draws random tensors and plants structure in them; it holds none of the
method's arithmetic (no pooling, scoring, selection or attention).

The workloads stand in for the long-context language-model workloads that
"Block Sparse Attention with Log-Linear Complexity" evaluates on (needle
retrieval at up to 256K tokens, §Experiments of its hyper.ai page); none of
that suite's items are reproduced. Recipe:

* every tensor is drawn in fp32 from its own ``torch.Generator`` seeded with
  ``seed + {0: q, 1: k, 2: v, 3: structure}``, structure is planted in fp32,
  then bf16 workloads are rounded once (round-to-nearest-even);
* ``needle``: for ``n_needles`` distinct query positions t ~ U[2C, N), a
  distinct earlier leaf block j < floor(t / C) gets keys
  4 * qhat + 0.3 * N(0, 1) in every kv head, qhat the unit vector of the sum
  of that head group's queries at t;
* ``clustered``: keys are a per-segment mean mu_s ~ N(0, I) (one per
  ``segment`` tokens and kv head) plus 0.5 * N(0, 1); q and v are N(0, 1);
* ``iid``: q, k, v ~ N(0, 1);
* ``periodic``: the keys of leaf i repeat those of leaf i mod ``period``
  (an N(0, 1) pattern of ``period`` leaves per kv head), so blocks of equal
  content recur and their scores tie exactly; q and v are N(0, 1).
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Prefill:
    name: str
    B: int
    N: int
    H_q: int
    H_kv: int
    d: int
    C: int
    K: int
    causal: bool
    dtype: str  # "f32" | "bf16"
    structure: str = "iid"  # "iid" | "needle" | "clustered"
    n_needles: int = 0
    segment: int = 4096
    period: int = 3
    seed: int = 0
    g: int = 2
    q_tile: int = 4

    @property
    def G_Q(self) -> int:
        return self.H_q // self.H_kv

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Prefill":
        return replace(self, **kw)


@dataclass(frozen=True)
class Decode:
    name: str
    S: int
    context: int
    steps: int
    H_q: int
    H_kv: int
    d: int
    C: int
    K: int
    dtype: str = "bf16"
    seed: int = 0
    g: int = 2

    @property
    def G_Q(self) -> int:
        return self.H_q // self.H_kv

    @property
    def cap(self) -> int:
        return self.context + self.steps

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Decode":
        return replace(self, **kw)


PREFILL = {
    "tiny_noncausal_1k": Prefill("tiny_noncausal_1k", B=1, N=1024, H_q=4, H_kv=1, d=64, C=32, K=4,
                                 causal=False, dtype="f32", seed=1000),
    "needle_16k": Prefill("needle_16k", B=1, N=16384, H_q=32, H_kv=8, d=128, C=64, K=16, causal=True,
                          dtype="bf16", structure="needle", n_needles=64, seed=2000),
    "clustered_64k": Prefill("clustered_64k", B=1, N=65536, H_q=32, H_kv=8, d=128, C=64, K=16, causal=True,
                             dtype="bf16", structure="clustered", segment=4096, seed=3000),
    "needle_256k": Prefill("needle_256k", B=1, N=262144, H_q=16, H_kv=2, d=128, C=64, K=16, causal=True,
                           dtype="bf16", structure="needle", n_needles=256, seed=4000),
    # The 256K head layout (G_Q = 8) at a quarter of the length: a profiling
    # and parity case for the G_Q = 8 kernels that still exceeds L2 (q: 268 MB).
    "needle_64k_g8": Prefill("needle_64k_g8", B=1, N=65536, H_q=16, H_kv=2, d=128, C=64, K=16, causal=True,
                             dtype="bf16", structure="needle", n_needles=64, seed=4500),
    # Half that again: q (134 MB) still exceeds L2, and the whole step fits in
    # about 2.5 GB of device memory, the size for single-kernel profiler captures.
    "needle_32k_g8": Prefill("needle_32k_g8", B=1, N=32768, H_q=16, H_kv=2, d=128, C=64, K=16, causal=True,
                             dtype="bf16", structure="needle", n_needles=32, seed=4600),
}

DECODE = {
    "decode_64x128k": Decode("decode_64x128k", S=64, context=131072, steps=256, H_q=32, H_kv=8, d=128, C=64,
                             K=16, dtype="bf16", seed=5000),
}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, device, seed: int) -> torch.Tensor:
    return torch.randn(shape, generator=_gen(device, seed), device=device, dtype=torch.float32)


def needle_placement(w: Prefill):
    """Positions t and leaf blocks j of the planted needles (CPU, seeded)."""
    g = _gen("cpu", w.seed + 3)
    lo = 2 * w.C
    if w.n_needles == 0 or w.N <= lo:
        return []
    n = min(w.n_needles, w.N - lo)
    ts = (torch.randperm(w.N - lo, generator=g)[:n] + lo).tolist()
    used = set()
    out = []
    for t in sorted(ts):
        own = t // w.C
        for _ in range(64):
            j = int(torch.randint(0, own, (1,), generator=g).item())
            if j not in used:
                used.add(j)
                out.append((t, j))
                break
    return out


def prefill_inputs(w: Prefill, device="cpu"):
    """q [B,H_q,N,d], k/v [B,H_kv,N,d] in the workload dtype, plus the needle list."""
    q = _randn((w.B, w.H_q, w.N, w.d), device, w.seed + 0)
    k = _randn((w.B, w.H_kv, w.N, w.d), device, w.seed + 1)
    v = _randn((w.B, w.H_kv, w.N, w.d), device, w.seed + 2)
    needles = []
    if w.structure == "needle":
        needles = needle_placement(w)
        g = _gen("cpu", w.seed + 4)
        for (t, j) in needles:
            lo, hi = j * w.C, min((j + 1) * w.C, w.N)
            for b in range(w.B):
                for h in range(w.H_kv):
                    qs = q[b, h * w.G_Q:(h + 1) * w.G_Q, t, :].sum(0)
                    qhat = qs / qs.norm()
                    noise = torch.randn((hi - lo, w.d), generator=g, dtype=torch.float32).to(device)
                    k[b, h, lo:hi, :] = 4.0 * qhat + 0.3 * noise
    elif w.structure == "clustered":
        nseg = (w.N + w.segment - 1) // w.segment
        mu = _randn((w.B, w.H_kv, nseg, w.d), device, w.seed + 3)
        k = 0.5 * k + mu.repeat_interleave(w.segment, dim=2)[:, :, : w.N, :]
    elif w.structure == "periodic":
        pat = k[:, :, : w.period * w.C, :]
        reps = -(-w.N // (w.period * w.C))
        k = pat.repeat(1, 1, reps, 1)[:, :, : w.N, :].contiguous()
    elif w.structure != "iid":
        raise ValueError(w.structure)
    dt = w.torch_dtype
    return dict(q=q.to(dt).contiguous(), k=k.to(dt).contiguous(), v=v.to(dt).contiguous(), needles=needles)


def decode_cache(w: Decode, device="cpu"):
    """K/V caches [S, H_kv, cap, d] holding ``context`` N(0,1) tokens per
    sequence (the rest zero), and the per-sequence lengths (int32)."""
    dt = w.torch_dtype
    kc = torch.zeros((w.S, w.H_kv, w.cap, w.d), dtype=dt, device=device)
    vc = torch.zeros((w.S, w.H_kv, w.cap, w.d), dtype=dt, device=device)
    for s in range(w.S):
        kc[s, :, : w.context] = torch.randn((w.H_kv, w.context, w.d), generator=_gen(device, w.seed + 16 * s + 1),
                                            device=device, dtype=torch.float32).to(dt)
        vc[s, :, : w.context] = torch.randn((w.H_kv, w.context, w.d), generator=_gen(device, w.seed + 16 * s + 2),
                                            device=device, dtype=torch.float32).to(dt)
    lens = torch.full((w.S,), w.context, dtype=torch.int32, device=device)
    return kc, vc, lens


def decode_step_inputs(w: Decode, step: int, device="cpu"):
    """New q [S,H_q,d], k/v [S,H_kv,d] for one decode step, seeded by step."""
    base = w.seed + 1_000_000 + 8 * step
    dt = w.torch_dtype
    q = _randn((w.S, w.H_q, w.d), device, base + 0).to(dt)
    k = _randn((w.S, w.H_kv, w.d), device, base + 1).to(dt)
    v = _randn((w.S, w.H_kv, w.d), device, base + 2).to(dt)
    return q, k, v
