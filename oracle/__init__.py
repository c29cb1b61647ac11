"""fp64 CPU oracle for the PISA hot path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package. The CUDA library never calls it, and the two share
no code: this package compiles ``pisa_oracle.cpp`` with g++ (no CUDA) and talks
to it through ctypes.

Every function follows a section of the hyper.ai page of "Block Sparse
Attention with Log-Linear Complexity" (the translated paper body); the C++
source cites the section at each step. Inputs are torch CPU tensors or numpy
arrays in their storage dtype (float32, or bfloat16 passed as raw 16-bit
patterns); all arithmetic is fp64.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, library routines on special cases, brute force on tiny inputs,
invariants and planted structure). Selection *quality* on real data is not
pinned (the pages print no numbers).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pisa_oracle.cpp")
_LIB = os.path.join(_HERE, "libpisa_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (OpenMP, fp64, no fast-math) if stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", _SRC, "-o", tmp]
        )
        os.replace(tmp, _LIB)
    return _LIB


class Cfg(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int64), ("N", ctypes.c_int64), ("H_q", ctypes.c_int64), ("H_kv", ctypes.c_int64),
        ("d", ctypes.c_int64), ("C", ctypes.c_int64), ("K", ctypes.c_int64), ("causal", ctypes.c_int64),
        ("dtype", ctypes.c_int64), ("Nq", ctypes.c_int64), ("q_t0", ctypes.c_int64), ("scale", ctypes.c_double),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            p = ctypes.c_void_p
            i64 = ctypes.c_int64
            lib.oracle_geometry.restype = i64
            lib.oracle_geometry.argtypes = [i64, i64, p, p]
            lib.oracle_build_pyramid.restype = None
            lib.oracle_build_pyramid.argtypes = [p, i64, i64, i64, i64, i64, i64, p]
            lib.oracle_select_rows.restype = None
            lib.oracle_select_rows.argtypes = [ctypes.POINTER(Cfg), p, p, p, i64, p, p, p, p, p, p, p]
            lib.oracle_select_flat_rows.restype = None
            lib.oracle_select_flat_rows.argtypes = [ctypes.POINTER(Cfg), p, p, i64, p, p, p]
            lib.oracle_select_exact_rows.restype = None
            lib.oracle_attn_bwd.restype = None
            lib.oracle_attn_bwd_dq_rows.restype = None
            lib.oracle_attn_bwd_dq_rows.argtypes = [ctypes.POINTER(Cfg), p, p, p, i64, p, p, p, p]
            lib.oracle_attn_bwd.argtypes = [ctypes.POINTER(Cfg), p, p, p, p, p, p, p, p]
            lib.oracle_select_exact_rows.argtypes = [ctypes.POINTER(Cfg), p, p, i64, p, p, p]
            lib.oracle_attn_rows.restype = None
            lib.oracle_attn_rows.argtypes = [ctypes.POINTER(Cfg), p, p, p, i64, p, p, p, p]
            lib.oracle_decode_append.restype = None
            lib.oracle_decode_append.argtypes = [p, i64, i64, i64, i64, i64, p]
            _lib = lib
    return _lib


def _storage(x):
    """Return (contiguous numpy array, dtype code) for a float32/bfloat16 tensor or array."""
    try:
        import torch
    except ImportError:  # pragma: no cover
        torch = None
    if torch is not None and isinstance(x, torch.Tensor):
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy(), 1
        if x.dtype == torch.float32:
            return x.numpy(), 0
        raise TypeError(f"oracle inputs must be float32 or bfloat16, got {x.dtype}")
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, 0
    if x.dtype in (np.int16, np.uint16):
        return x, 1
    raise TypeError(f"oracle inputs must be float32 or bf16 bit patterns, got {x.dtype}")


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def geometry(N: int, C: int):
    """Level sizes M[0..L] (M[0] = N raw keys) and level row offsets off[0..L]
    (level l starts at off[l-1], off[L] = rows per head). §Pyramid level sizes."""
    lib = _load()
    L = lib.oracle_geometry(N, C, None, None)
    sizes = np.zeros(L + 1, np.int64)
    offs = np.zeros(L + 1, np.int64)
    lib.oracle_geometry(N, C, _ptr(sizes), _ptr(offs))
    return sizes, offs


def build_pyramid(k, C: int) -> np.ndarray:
    """Mean-pooled pyramid of k [B, H, N, d] -> fp64 [B, H, R, d] (§Pyramid)."""
    a, code = _storage(k)
    B, H, N, d = a.shape
    _, offs = geometry(N, C)
    out = np.zeros((B, H, int(offs[-1]), d), np.float64)
    _load().oracle_build_pyramid(_ptr(a), code, B, H, N, d, C, _ptr(out))
    return out


def make_cfg(*, B, N, H_q, H_kv, d, C, K, causal, dtype_code, scale=0.0, Nq=None, q_t0=0) -> Cfg:
    return Cfg(B, N, H_q, H_kv, d, C, K, int(bool(causal)), dtype_code, N if Nq is None else Nq, q_t0, scale)


def _rows(rows) -> np.ndarray:
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    return r


def select_rows(cfg: Cfg, q, k, pyr: np.ndarray, rows, trace: bool = False):
    """Coarse-to-fine top-K (§TopK) for rows (b, kv head, t).

    Returns sel [n, K] int32 (ascending, -1 padded) and min_gap [n] (smallest
    K-th minus (K+1)-th score over the scored levels; inf if none), plus, with
    ``trace``, per-level candidate counts, candidates, scores and kept flags.
    """
    qa, _ = _storage(q)
    ka, _ = _storage(k)
    pyr = np.ascontiguousarray(pyr, dtype=np.float64)
    r = _rows(rows)
    n = r.shape[0]
    K = cfg.K
    sel = np.zeros((n, K), np.int32)
    gap = np.zeros(n, np.float64)
    lib = _load()
    if trace:
        L = len(geometry(cfg.N, cfg.C)[0]) - 1
        W = 2 * K
        tn = np.zeros((n, L + 1), np.int32)
        tc = np.full((n, L + 1, W), -1, np.int32)
        ts = np.full((n, L + 1, W), np.nan, np.float64)
        tk = np.zeros((n, L + 1, W), np.uint8)
        lib.oracle_select_rows(ctypes.byref(cfg), _ptr(qa), _ptr(ka), _ptr(pyr), n, _ptr(r), _ptr(sel), _ptr(gap),
                               _ptr(tn), _ptr(tc), _ptr(ts), _ptr(tk))
        return sel, gap, dict(n=tn, cand=tc, score=ts, kept=tk.astype(bool))
    lib.oracle_select_rows(ctypes.byref(cfg), _ptr(qa), _ptr(ka), _ptr(pyr), n, _ptr(r), _ptr(sel), _ptr(gap),
                           None, None, None, None)
    return sel, gap


def select_flat_rows(cfg: Cfg, q, pyr: np.ndarray, rows):
    """Flat single-level selector (§BSA, flat block scoring) for rows (b, kv head, t)."""
    qa, _ = _storage(q)
    pyr = np.ascontiguousarray(pyr, dtype=np.float64)
    r = _rows(rows)
    n = r.shape[0]
    sel = np.zeros((n, cfg.K), np.int32)
    gap = np.zeros(n, np.float64)
    _load().oracle_select_flat_rows(ctypes.byref(cfg), _ptr(qa), _ptr(pyr), n, _ptr(r), _ptr(sel), _ptr(gap))
    return sel, gap


def select_exact_rows(cfg: Cfg, q, k, rows):
    """Exact-score flat selector (every usable leaf scored by its raw-key LSE,
    summed over the GQA group) for rows (b, kv head, t). Returns sel [n, K]
    and the K-th minus (K+1)-th score gap per row (inf when kept unscored)."""
    qa, _ = _storage(q)
    ka, _ = _storage(k)
    r = _rows(rows)
    n = r.shape[0]
    sel = np.zeros((n, cfg.K), np.int32)
    gap = np.zeros(n, np.float64)
    _load().oracle_select_exact_rows(ctypes.byref(cfg), _ptr(qa), _ptr(ka), n, _ptr(r), _ptr(sel), _ptr(gap))
    return sel, gap


def attn_rows(cfg: Cfg, q, k, v, rows, sel):
    """Block-sparse attention (§BSA) for rows (b, kv head, t) over the given
    selections sel [n, K]. Returns out [n, G, d] and lse [n, G], fp64."""
    qa, _ = _storage(q)
    ka, _ = _storage(k)
    va, _ = _storage(v)
    r = _rows(rows)
    n = r.shape[0]
    G = cfg.H_q // cfg.H_kv
    s = np.ascontiguousarray(np.asarray(sel, dtype=np.int32).reshape(n, cfg.K))
    out = np.zeros((n, G, cfg.d), np.float64)
    lse = np.zeros((n, G), np.float64)
    _load().oracle_attn_rows(ctypes.byref(cfg), _ptr(qa), _ptr(ka), _ptr(va), n, _ptr(r), _ptr(s), _ptr(out), _ptr(lse))
    return out, lse


def attn_bwd(cfg: Cfg, q, k, v, sel, dout):
    """Gradient of the block-sparse attention with the selection sel
    [B, H_kv, N, K] held fixed: returns dq [B, H_q, N, d], dk, dv
    [B, H_kv, N, d] (fp64) for the output gradient dout [B, H_q, N, d]."""
    qa, _ = _storage(q)
    ka, _ = _storage(k)
    va, _ = _storage(v)
    ga, _ = _storage(dout)
    s = np.ascontiguousarray(np.asarray(sel, dtype=np.int32))
    dq = np.zeros((cfg.B, cfg.H_q, cfg.N, cfg.d), np.float64)
    dk = np.zeros((cfg.B, cfg.H_kv, cfg.N, cfg.d), np.float64)
    dv = np.zeros((cfg.B, cfg.H_kv, cfg.N, cfg.d), np.float64)
    _load().oracle_attn_bwd(ctypes.byref(cfg), _ptr(qa), _ptr(ka), _ptr(va), _ptr(s), _ptr(ga), _ptr(dq), _ptr(dk),
                            _ptr(dv))
    return dq, dk, dv


def attn_bwd_dq_rows(cfg: Cfg, q, k, v, rows, sel, dout):
    """dq of the attention backward for rows (b, kv head, t) only, given their
    selections sel [n, K]: returns [n, G, d] fp64."""
    qa, _ = _storage(q)
    ka, _ = _storage(k)
    va, _ = _storage(v)
    ga, _ = _storage(dout)
    r = _rows(rows)
    n = r.shape[0]
    G = cfg.H_q // cfg.H_kv
    s = np.ascontiguousarray(np.asarray(sel, dtype=np.int32).reshape(n, cfg.K))
    dq = np.zeros((n, G, cfg.d), np.float64)
    _load().oracle_attn_bwd_dq_rows(ctypes.byref(cfg), _ptr(qa), _ptr(ka), _ptr(va), n, _ptr(r), _ptr(s), _ptr(ga),
                                    _ptr(dq))
    return dq


def decode_append(seq_keys, n: int, C: int, cap: int, pyr: np.ndarray) -> None:
    """In-place decode update of one sequence's capacity-laid-out fp64 pyramid
    after key n was appended (§Kernels, decoding). seq_keys: [>= n+1, d]."""
    a, code = _storage(seq_keys)
    d = a.shape[-1]
    assert pyr.dtype == np.float64 and pyr.flags.c_contiguous
    _load().oracle_decode_append(_ptr(a), code, n, d, C, cap, _ptr(pyr))
