"""Shared helpers for the GPU-vs-oracle parity tests.

Acceptance (the problem statement's tolerances):
  * pyramid geometry bit-exact; summaries within 1e-5 + 1e-6 |x| of fp64;
  * selected sets identical except on rows whose oracle gap between the K-th
    and (K+1)-th summed score is below 1e-3 at some scored level (exempt);
  * attention max-abs error <= 2e-2 for bf16 I/O, <= 1e-4 for fp32, with the
    GPU's own selection fed to the oracle; lse within 1e-3 (bf16) / 1e-4 (fp32).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O

GAP_TOL = 1e-3
ATTN_TOL = {"bf16": 2e-2, "f32": 1e-4}
LSE_TOL = {"bf16": 1e-3, "f32": 1e-4}


def dtype_code(w):
    return 0 if w.dtype == "f32" else 1


def ocfg(w, **kw):
    return O.make_cfg(B=w.B, N=w.N, H_q=w.H_q, H_kv=w.H_kv, d=w.d, C=w.C, K=w.K, causal=w.causal,
                      dtype_code=dtype_code(w), **kw)


def host(x: torch.Tensor) -> torch.Tensor:
    return x.detach().cpu().contiguous()


def sample_rows(w, n_per_head: int | None, seed: int = 0, extra_t=()):
    """(b, h, t) rows: all rows when n_per_head is None, else a seeded sample
    per (b, h) plus the first and last two leaves' positions and extra_t."""
    if n_per_head is None or n_per_head >= w.N:
        ts = np.arange(w.N)
    else:
        rng = np.random.default_rng(seed)
        edge = list(range(0, min(2 * w.C, w.N))) + list(range(max(0, w.N - 2 * w.C), w.N))
        ts = np.unique(np.concatenate([rng.choice(w.N, n_per_head, replace=False), edge,
                                       np.asarray(list(extra_t), dtype=np.int64)]).astype(np.int64))
    return np.array([(b, h, t) for b in range(w.B) for h in range(w.H_kv) for t in ts], dtype=np.int64)


def check_pyramid(w, k_host, pyr_gpu_host):
    ref = O.build_pyramid(k_host, w.C)
    got = pyr_gpu_host.numpy().astype(np.float64)
    assert got.shape == ref.shape
    err = np.abs(got - ref)
    bound = 1e-5 + 1e-6 * np.abs(ref)
    assert (err <= bound).all(), f"pyramid max err {err.max():.3e}"
    return ref


def compare_selection(w, sel_gpu_rows: np.ndarray, sel_ref: np.ndarray, gap: np.ndarray):
    """Returns (n_rows, n_exempt, n_mismatch_nonexempt, n_mismatch_exempt)."""
    same = (np.sort(sel_gpu_rows, 1) == np.sort(sel_ref, 1)).all(1)
    exempt = gap < GAP_TOL
    return len(same), int(exempt.sum()), int((~same & ~exempt).sum()), int((~same & exempt).sum())


def check_attention(w, out_gpu_rows: np.ndarray, lse_gpu_rows: np.ndarray | None, out_ref, lse_ref):
    err = np.abs(out_gpu_rows.astype(np.float64) - out_ref)
    tol = ATTN_TOL[w.dtype]
    assert err.max() <= tol, f"attention max-abs err {err.max():.3e} > {tol}"
    if lse_gpu_rows is not None:
        lerr = np.abs(lse_gpu_rows.astype(np.float64) - lse_ref)
        assert lerr.max() <= LSE_TOL[w.dtype], f"lse max err {lerr.max():.3e}"
    return float(err.max())


def gather_rows(sel: torch.Tensor, rows: np.ndarray) -> np.ndarray:
    """sel [B, H_kv, N, K] -> [n, K] at the given (b, h, t) rows."""
    s = host(sel).numpy()
    return s[rows[:, 0], rows[:, 1], rows[:, 2]]


def gather_out(w, out: torch.Tensor, rows: np.ndarray) -> np.ndarray:
    """out [B, H_q, N, d] -> [n, G, d] at the given (b, kv head, t) rows."""
    o = host(out).float().numpy()
    G = w.H_q // w.H_kv
    hq = rows[:, 1:2] * G + np.arange(G)[None, :]
    return o[rows[:, 0:1], hq, rows[:, 2:3], :]


def gather_lse(w, lse: torch.Tensor, rows: np.ndarray) -> np.ndarray:
    s = host(lse).numpy()
    G = w.H_q // w.H_kv
    hq = rows[:, 1:2] * G + np.arange(G)[None, :]
    return s[rows[:, 0:1], hq, rows[:, 2:3]]
