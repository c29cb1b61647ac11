"""Public Python API over the C ABI (include/pisa.h).

PyTorch supplies device memory and streams; every computation runs in the
library's CUDA kernels. Tensors must be contiguous CUDA tensors in bfloat16
or float32 ([B, H, N, d] for q/k/v); results are written into the given (or
newly allocated) output tensors on the current stream.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass

import torch

from . import _lib

_DT = {torch.float32: _lib.DTYPE_F32, torch.bfloat16: _lib.DTYPE_BF16}


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None, shape=None):
    """Checks a tensor handed to the library: the kernels trust every size, so
    a buffer of the wrong shape would be read or written out of bounds."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    _on_cuda(t, name)


def _on_cuda(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    _check_device_index(t.device.index, name)


def _check_device_index(index, name: str):
    """The C library launches on the runtime's current device, so every tensor
    of a call must live there: another GPU's pointers would reach the kernels
    and their TMA descriptors. Make the tensors' device current first
    (torch.cuda.set_device or a torch.cuda.device(...) block)."""
    cur = torch.cuda.current_device()
    if index is not None and index != cur:
        raise ValueError(f"{name} is on cuda:{index} but the current device is cuda:{cur}; "
                         f"call under torch.cuda.device({index})")


def launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(_lib.lib().pisa_launch_count())


def device_faults() -> int:
    """Bounded device waits that ran out of time on the current device (synchronises)."""
    return int(_lib.lib().pisa_device_faults())


class KernelTimer:
    """Per-kernel device time of every library launch inside a ``with`` block
    (pisa_timing_start / pisa_timing_stop): CUDA events on each launching
    stream. On exit, ``result`` maps kernel name -> (total ms, launches).
    Exiting synchronises with the timed streams."""

    MAX = 64

    def __enter__(self):
        _lib.call("pisa_timing_start")
        self.result = {}
        return self

    def __exit__(self, *exc):
        names = (ctypes.c_char_p * self.MAX)()
        ms = (ctypes.c_double * self.MAX)()
        cnt = (ctypes.c_int * self.MAX)()
        n = _lib.lib().pisa_timing_stop(self.MAX, names, ms, cnt)
        if n < 0:
            raise RuntimeError("pisa_timing_stop: a timing event failed")
        self.result = {names[i].decode(): (ms[i], cnt[i]) for i in range(min(n, self.MAX))}
        return False


def pyramid_geometry(N: int, C: int, g: int = 2):
    """(L, offsets): level l (1..L) occupies rows offsets[l-1]:offsets[l]."""
    L = ctypes.c_int32()
    _lib.call("pisa_pyramid_geometry", N, C, g, ctypes.byref(L), None)
    offs = (ctypes.c_int64 * (L.value + 1))()
    _lib.call("pisa_pyramid_geometry", N, C, g, ctypes.byref(L), offs)
    return L.value, list(offs)


def pyramid_rows(N: int, C: int) -> int:
    return int(_lib.lib().pisa_pyramid_rows(N, C))


@dataclass(frozen=True)
class Problem:
    """Prefill shape and hyper-parameters (paper: C leaf size, g = 2, K, Q_tile = 4)."""
    B: int
    N: int
    H_q: int
    H_kv: int
    d: int
    C: int
    K: int
    causal: bool
    dtype: torch.dtype
    scale: float = 0.0
    g: int = 2
    q_tile: int = 4

    @staticmethod
    def of(q: torch.Tensor, k: torch.Tensor, *, C: int, K: int, causal: bool, scale: float = 0.0) -> "Problem":
        B, H_q, N, d = q.shape
        Bk, H_kv, Nk, dk = k.shape
        if (B, N, d) != (Bk, Nk, dk):
            raise ValueError(f"q {tuple(q.shape)} and k {tuple(k.shape)} disagree")
        if q.dtype != k.dtype or q.dtype not in _DT:
            raise ValueError("q and k must share dtype float32 or bfloat16")
        return Problem(B, N, H_q, H_kv, d, C, K, bool(causal), q.dtype, scale)

    def cstruct(self) -> _lib.Config:
        return _lib.Config(self.B, self.N, self.H_q, self.H_kv, self.d, self.C, self.g, self.K, self.q_tile,
                           int(self.causal), _DT[self.dtype], self.scale)

    @property
    def R(self) -> int:
        return pyramid_rows(self.N, self.C)

    def workspace_bytes(self) -> int:
        return int(_lib.lib().pisa_select_workspace_bytes(ctypes.byref(self.cstruct())))


def build_pyramid(k: torch.Tensor, *, C: int, out: torch.Tensor | None = None) -> torch.Tensor:
    """Mean-pooled key pyramid of k [B, H_kv, N, d] -> fp32 [B, H_kv, R, d]."""
    _need(k, "k")
    B, H, N, d = k.shape
    pr = Problem(B, N, H, H, d, C, 1, False, k.dtype)
    if out is None:
        out = torch.empty((B, H, pr.R, d), dtype=torch.float32, device=k.device)
    _need(out, "out", torch.float32, (B, H, pr.R, d))
    _lib.call("pisa_build_pyramid", ctypes.byref(pr.cstruct()), _p(k), _p(out), _stream(k))
    return out


def select(q, k, pyr, *, C: int, K: int, causal: bool, scale: float = 0.0, out=None, score=None,
           workspace=None):
    """PISA coarse-to-fine top-K leaf blocks: sel [B, H_kv, N, K] int32 (ascending, -1 padded)."""
    _need(q, "q")
    _need(k, "k", q.dtype)
    pr = Problem.of(q, k, C=C, K=K, causal=causal, scale=scale)
    _need(pyr, "pyr", torch.float32, (pr.B, pr.H_kv, pr.R, pr.d))
    rows = (pr.B, pr.H_kv, pr.N, K)
    if out is None:
        out = torch.empty(rows, dtype=torch.int32, device=q.device)
    _need(out, "out", torch.int32, rows)
    if score is not None:
        _need(score, "score", torch.float32, rows)
    need = pr.workspace_bytes()
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace")
    _lib.call("pisa_select", ctypes.byref(pr.cstruct()), _p(q), _p(k), _p(pyr), _p(out), _p(score), _p(workspace),
              workspace.numel() * workspace.element_size(), _stream(q))
    return out


def select_flat(q, pyr, *, C: int, K: int, causal: bool, H_kv: int, scale: float = 0.0, out=None,
                workspace=None):
    """Flat single-level top-K over all leaf summaries: sel [B, H_kv, N, K] int32."""
    _need(q, "q")
    B, H_q, N, d = q.shape
    pr = Problem(B, N, H_q, H_kv, d, C, K, bool(causal), q.dtype, scale)
    _need(pyr, "pyr", torch.float32, (B, H_kv, pr.R, d))
    if out is None:
        out = torch.empty((B, H_kv, N, K), dtype=torch.int32, device=q.device)
    _need(out, "out", torch.int32, (B, H_kv, N, K))
    need = int(_lib.lib().pisa_select_flat_workspace_bytes(ctypes.byref(pr.cstruct())))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace")
    _lib.call("pisa_select_flat", ctypes.byref(pr.cstruct()), _p(q), _p(pyr), _p(out), _p(workspace),
              workspace.numel() * workspace.element_size(), _stream(q))
    return out


def sparse_attn_bwd(q, k, v, sel, out, lse, dout, *, C: int, causal: bool, scale: float = 0.0):
    """Gradients (dq, dk, dv; fp32) of the block-sparse attention with the
    selection sel held fixed, for the output gradient dout; out and lse are the
    forward's outputs. bf16 inputs."""
    _need(q, "q")
    _need(k, "k", q.dtype)
    _need(v, "v", q.dtype, k.shape)
    _need(out, "out", q.dtype, q.shape)
    _need(dout, "dout", q.dtype, q.shape)
    pr = Problem.of(q, k, C=C, K=sel.shape[-1], causal=causal, scale=scale)
    _need(sel, "sel", torch.int32, (pr.B, pr.H_kv, pr.N, pr.K))
    _need(lse, "lse", torch.float32, (pr.B, pr.H_q, pr.N))
    cfg = pr.cstruct()
    nbytes = int(_lib.lib().pisa_attn_bwd_workspace_bytes(ctypes.byref(cfg)))
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
    _lib.call("pisa_sparse_attn_bwd", ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(sel), _p(out), _p(lse), _p(dout),
              _p(dq), _p(dk), _p(dv), _p(ws), ws.numel(), _stream(q))
    return dq, dk, dv


def select_exact(q, k, *, C: int, K: int, causal: bool, scale: float = 0.0, out=None):
    """Exact-score flat top-K: every usable leaf scored by its raw-key LSE
    summed over the group. sel [B, H_kv, N, K] int32."""
    _need(q, "q")
    _need(k, "k", q.dtype)
    pr = Problem.of(q, k, C=C, K=K, causal=causal, scale=scale)
    if out is None:
        out = torch.empty((pr.B, pr.H_kv, pr.N, K), dtype=torch.int32, device=q.device)
    _need(out, "out", torch.int32, (pr.B, pr.H_kv, pr.N, K))
    _lib.call("pisa_select_exact", ctypes.byref(pr.cstruct()), _p(q), _p(k), _p(out), _stream(q))
    return out


def _attn_workspace(cfg, span, device, workspace):
    """The caller's workspace, or a new one of the size the bucketed
    attention needs (None when that route does not apply)."""
    if workspace is not None:
        _need(workspace, "workspace")
        return workspace
    need = int(_lib.lib().pisa_attn_fwd_span_workspace_bytes(ctypes.byref(cfg), ctypes.byref(span)))
    return torch.empty(need, dtype=torch.uint8, device=device) if need > 0 else None


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def sparse_attn_fwd(q, k, v, sel, *, C: int, causal: bool, scale: float = 0.0, out=None, lse=None,
                    want_lse: bool = True, workspace=None):
    """Block-sparse attention over the selected leaf blocks: (out [B,H_q,N,d], lse [B,H_q,N] or None).
    The bucketed route's scratch is allocated here unless `workspace` is given."""
    _need(q, "q")
    _need(k, "k", q.dtype)
    _need(v, "v", q.dtype, k.shape)
    pr = Problem.of(q, k, C=C, K=sel.shape[-1], causal=causal, scale=scale)
    _need(sel, "sel", torch.int32, (pr.B, pr.H_kv, pr.N, pr.K))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", q.dtype, q.shape)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, q.shape[:-1])
    cfg = pr.cstruct()
    ws = _attn_workspace(cfg, _lib.QuerySpan(0, pr.N), q.device, workspace)
    _lib.call("pisa_sparse_attn_fwd", ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(sel), _p(out), _p(lse), _p(ws),
              _nbytes(ws), _stream(q))
    return out, lse


def _span_problem(q, k, C, K, causal, scale):
    B, H_q, n_q, d = q.shape
    Bk, H_kv, N, dk = k.shape
    if (B, d) != (Bk, dk) or q.dtype != k.dtype or q.dtype not in _DT:
        raise ValueError(f"q {tuple(q.shape)} {q.dtype} and k {tuple(k.shape)} {k.dtype} disagree")
    return Problem(B, N, H_q, H_kv, d, C, K, bool(causal), q.dtype, scale), n_q


def select_span(q, k, pyr, *, q0: int, C: int, K: int, causal: bool, scale: float = 0.0, out=None, score=None,
                workspace=None):
    """Selection for the query rows at positions [q0, q0 + n_q) of a sequence:
    q [B, H_q, n_q, d] holds those rows only; k [B, H_kv, N, d] and pyr cover
    all N tokens. Returns sel [B, H_kv, n_q, K], equal to those rows of a
    whole-sequence selection."""
    _need(q, "q")
    _need(k, "k", q.dtype)
    pr, n_q = _span_problem(q, k, C, K, causal, scale)
    _need(pyr, "pyr", torch.float32, (pr.B, pr.H_kv, pr.R, pr.d))
    cfg, span = pr.cstruct(), _lib.QuerySpan(q0, n_q)
    rows = (pr.B, pr.H_kv, n_q, K)
    if out is None:
        out = torch.empty(rows, dtype=torch.int32, device=q.device)
    _need(out, "out", torch.int32, rows)
    if score is not None:
        _need(score, "score", torch.float32, rows)
    if workspace is None:
        need = int(_lib.lib().pisa_select_span_workspace_bytes(ctypes.byref(cfg), ctypes.byref(span)))
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace")
    _lib.call("pisa_select_span", ctypes.byref(cfg), ctypes.byref(span), _p(q), _p(k), _p(pyr), _p(out), _p(score),
              _p(workspace), workspace.numel() * workspace.element_size(), _stream(q))
    return out


def sparse_attn_fwd_span(q, k, v, sel, *, q0: int, C: int, causal: bool, scale: float = 0.0, out=None, lse=None,
                         want_lse: bool = True, workspace=None):
    """Block-sparse attention for the query rows at positions [q0, q0 + n_q):
    q [B, H_q, n_q, d] and sel [B, H_kv, n_q, K] hold those rows; k and v all
    N tokens. Returns (out [B, H_q, n_q, d], lse [B, H_q, n_q] or None)."""
    _need(q, "q")
    _need(k, "k", q.dtype)
    _need(v, "v", q.dtype, k.shape)
    pr, n_q = _span_problem(q, k, C, sel.shape[-1], causal, scale)
    _need(sel, "sel", torch.int32, (pr.B, pr.H_kv, n_q, pr.K))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", q.dtype, q.shape)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, q.shape[:-1])
    cfg, span = pr.cstruct(), _lib.QuerySpan(q0, n_q)
    ws = _attn_workspace(cfg, span, q.device, workspace)
    _lib.call("pisa_sparse_attn_fwd_span", ctypes.byref(cfg), ctypes.byref(span), _p(q), _p(k), _p(v), _p(sel),
              _p(out), _p(lse), _p(ws), _nbytes(ws), _stream(q))
    return out, lse


class Prefill:
    """Reusable prefill pipeline for one problem shape: pyramid, PISA select
    and block-sparse attention, with all buffers allocated once. Calling it
    checks q, k and v against the problem. The stage methods (pyramid,
    select, attend) skip that check and expect the problem's shapes."""

    def __init__(self, pr: Problem, device="cuda"):
        self.pr = pr
        dev = torch.device(device)
        self.cfg = pr.cstruct()
        self.pyr = torch.empty((pr.B, pr.H_kv, pr.R, pr.d), dtype=torch.float32, device=dev)
        self.sel = torch.empty((pr.B, pr.H_kv, pr.N, pr.K), dtype=torch.int32, device=dev)
        # One scratch buffer serves the selection and then the attention (the
        # selection's scratch is dead once sel is written).
        self.attn_ws_bytes = int(_lib.lib().pisa_attn_fwd_workspace_bytes(ctypes.byref(self.cfg)))
        self.ws = torch.empty(max(pr.workspace_bytes(), self.attn_ws_bytes, 256), dtype=torch.uint8, device=dev)
        self.out = torch.empty((pr.B, pr.H_q, pr.N, pr.d), dtype=pr.dtype, device=dev)
        self.lse = torch.empty((pr.B, pr.H_q, pr.N), dtype=torch.float32, device=dev)

    def pyramid(self, k):
        _lib.call("pisa_build_pyramid", ctypes.byref(self.cfg), _p(k), _p(self.pyr), _stream(k))

    def select(self, q, k):
        _lib.call("pisa_select", ctypes.byref(self.cfg), _p(q), _p(k), _p(self.pyr), _p(self.sel), None,
                  _p(self.ws), self.ws.numel(), _stream(q))

    def attend(self, q, k, v):
        ws = self.ws if self.attn_ws_bytes else None
        _lib.call("pisa_sparse_attn_fwd", ctypes.byref(self.cfg), _p(q), _p(k), _p(v), _p(self.sel), _p(self.out),
                  _p(self.lse), _p(ws), _nbytes(ws), _stream(q))

    def check(self, q, k, v):
        """Raises unless q, k and v have this problem's shapes and dtype."""
        pr = self.pr
        _need(q, "q", pr.dtype, (pr.B, pr.H_q, pr.N, pr.d))
        _need(k, "k", pr.dtype, (pr.B, pr.H_kv, pr.N, pr.d))
        _need(v, "v", pr.dtype, (pr.B, pr.H_kv, pr.N, pr.d))

    def __call__(self, q, k, v):
        self.check(q, k, v)
        self.pyramid(k)
        self.select(q, k)
        self.attend(q, k, v)
        return self.out


class PrefillShard:
    """Prefill of the query rows at positions [q0, q0 + n_q) of an N-token
    sequence (pr describes the whole sequence): the pyramid over all N keys,
    then the selection and attention of this shard's rows only, with buffers
    allocated once. q is [B, H_q, n_q, d]; k and v are [B, H_kv, N, d].
    Calling it checks them; the stage methods do not."""

    def __init__(self, pr: Problem, q0: int, n_q: int, device="cuda"):
        self.pr, self.q0, self.n_q = pr, q0, n_q
        dev = torch.device(device)
        self.cfg = pr.cstruct()
        self.span = _lib.QuerySpan(q0, n_q)
        nbytes = int(_lib.lib().pisa_select_span_workspace_bytes(ctypes.byref(self.cfg), ctypes.byref(self.span)))
        if pr.dtype == torch.bfloat16 and nbytes == 0:
            raise ValueError(f"query span [{q0}, {q0 + n_q}) does not fit N = {pr.N}")
        self.pyr = torch.empty((pr.B, pr.H_kv, pr.R, pr.d), dtype=torch.float32, device=dev)
        self.sel = torch.empty((pr.B, pr.H_kv, n_q, pr.K), dtype=torch.int32, device=dev)
        self.attn_ws_bytes = int(_lib.lib().pisa_attn_fwd_span_workspace_bytes(ctypes.byref(self.cfg),
                                                                               ctypes.byref(self.span)))
        self.ws = torch.empty(max(nbytes, self.attn_ws_bytes, 256), dtype=torch.uint8, device=dev)
        self.out = torch.empty((pr.B, pr.H_q, n_q, pr.d), dtype=pr.dtype, device=dev)
        self.lse = torch.empty((pr.B, pr.H_q, n_q), dtype=torch.float32, device=dev)

    def pyramid(self, k):
        _lib.call("pisa_build_pyramid", ctypes.byref(self.cfg), _p(k), _p(self.pyr), _stream(k))

    def select(self, q, k):
        _lib.call("pisa_select_span", ctypes.byref(self.cfg), ctypes.byref(self.span), _p(q), _p(k), _p(self.pyr),
                  _p(self.sel), None, _p(self.ws), self.ws.numel(), _stream(q))

    def attend(self, q, k, v):
        ws = self.ws if self.attn_ws_bytes else None
        _lib.call("pisa_sparse_attn_fwd_span", ctypes.byref(self.cfg), ctypes.byref(self.span), _p(q), _p(k), _p(v),
                  _p(self.sel), _p(self.out), _p(self.lse), _p(ws), _nbytes(ws), _stream(q))

    def check(self, q, k, v):
        """Raises unless q holds this shard's rows and k, v the whole sequence."""
        pr = self.pr
        _need(q, "q", pr.dtype, (pr.B, pr.H_q, self.n_q, pr.d))
        _need(k, "k", pr.dtype, (pr.B, pr.H_kv, pr.N, pr.d))
        _need(v, "v", pr.dtype, (pr.B, pr.H_kv, pr.N, pr.d))

    def __call__(self, q, k, v):
        self.check(q, k, v)
        self.pyramid(k)
        self.select(q, k)
        self.attend(q, k, v)
        return self.out


def prefill(q, k, v, *, C: int, K: int, causal: bool, scale: float = 0.0):
    """Pyramid + PISA selection + block-sparse attention in one call: (out, lse, sel)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
    p = Prefill(Problem.of(q, k, C=C, K=K, causal=causal, scale=scale), q.device)
    p(q, k, v)
    return p.out, p.lse, p.sel


class PrefillStream:
    """Prefill steps over batches held in pinned host memory, with the
    host-device copies overlapped with compute.

    While step s computes on the current stream, step s + 1's q, k and v are
    copied in on one copy stream, and step s - 1's output is copied out on
    another. Each step uses one of `depth` slots: device inputs plus a
    Prefill pipeline with its own outputs. Events order the slots, so a slot
    is refilled only after its previous step has computed, and recomputed
    only after its previous output has been copied out.

    The host tensors passed to submit() must stay alive and unchanged until
    that step's output copy has finished (synchronize(), or the returned
    event)."""

    def __init__(self, pr: Problem, device="cuda", depth: int = 2):
        if depth < 1:
            raise ValueError("depth must be at least 1")
        dev = torch.device(device)
        self.pr, self.dev = pr, dev
        self.h2d = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)
        self.slots = []
        for _ in range(depth):
            self.slots.append({
                "p": Prefill(pr, dev),
                "q": torch.empty((pr.B, pr.H_q, pr.N, pr.d), dtype=pr.dtype, device=dev),
                "k": torch.empty((pr.B, pr.H_kv, pr.N, pr.d), dtype=pr.dtype, device=dev),
                "v": torch.empty((pr.B, pr.H_kv, pr.N, pr.d), dtype=pr.dtype, device=dev),
                "loaded": torch.cuda.Event(), "computed": torch.cuda.Event(), "drained": torch.cuda.Event(),
            })
        # The copy streams use these buffers. If this object is dropped with
        # copies still queued, the allocator must not hand the memory to a
        # new tensor until they finish.
        for slot in self.slots:
            for name in ("q", "k", "v"):
                slot[name].record_stream(self.h2d)
            slot["p"].out.record_stream(self.d2h)
        self.steps = 0

    def submit(self, hq, hk, hv, hout):
        """Enqueues one step: hq, hk, hv (pinned host [B, H, N, d]) in, the
        prefill, its output into hout (pinned host [B, H_q, N, d]). Returns
        the event that completes when hout holds the output."""
        pr = self.pr
        for t, name, H in ((hq, "q", pr.H_q), (hk, "k", pr.H_kv), (hv, "v", pr.H_kv), (hout, "out", pr.H_q)):
            if t.is_cuda or not t.is_pinned() or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous tensor in pinned host memory")
            if t.dtype != pr.dtype or tuple(t.shape) != (pr.B, H, pr.N, pr.d):
                raise ValueError(f"{name} must be {pr.dtype} [{pr.B}, {H}, {pr.N}, {pr.d}]")
        slot = self.slots[self.steps % len(self.slots)]
        self.steps += 1
        compute = torch.cuda.current_stream(self.dev)
        self.h2d.wait_event(slot["computed"])  # the slot's previous step has read its inputs
        with torch.cuda.stream(self.h2d):
            slot["q"].copy_(hq, non_blocking=True)
            slot["k"].copy_(hk, non_blocking=True)
            slot["v"].copy_(hv, non_blocking=True)
            slot["loaded"].record(self.h2d)
        compute.wait_event(slot["loaded"])
        compute.wait_event(slot["drained"])  # the slot's previous output has been copied out
        slot["p"](slot["q"], slot["k"], slot["v"])
        slot["computed"].record(compute)
        self.d2h.wait_event(slot["computed"])
        with torch.cuda.stream(self.d2h):
            hout.copy_(slot["p"].out, non_blocking=True)
            slot["drained"].record(self.d2h)
        return slot["drained"]

    def synchronize(self):
        """Waits on the host until every submitted step's output is in host memory."""
        self.d2h.synchronize()


class DecodeState:
    """Caller-side decode state for S sequences of capacity cap: KV caches,
    the cached mean pyramid, per-sequence lengths, a device status word and
    the decode workspace."""

    def __init__(self, *, S: int, cap: int, H_q: int, H_kv: int, d: int, C: int, K: int,
                 dtype=torch.bfloat16, scale: float = 0.0, device="cuda", k_cache=None, v_cache=None, lens=None):
        dev = torch.device(device)
        self.cfg = _lib.DecodeConfig(S, cap, H_q, H_kv, d, C, 2, K, _DT[dtype], scale)
        self.S, self.cap, self.H_q, self.H_kv, self.d, self.C, self.K = S, cap, H_q, H_kv, d, C, K
        self.dtype = dtype
        R = int(_lib.lib().pisa_decode_pyramid_rows(ctypes.byref(self.cfg)))
        if R <= 0:
            raise _lib.PisaError("pisa_decode_pyramid_rows", 1)
        self.R = R
        self.k_cache = k_cache if k_cache is not None else torch.zeros((S, H_kv, cap, d), dtype=dtype, device=dev)
        self.v_cache = v_cache if v_cache is not None else torch.zeros((S, H_kv, cap, d), dtype=dtype, device=dev)
        self.len = lens if lens is not None else torch.zeros(S, dtype=torch.int32, device=dev)
        for t, n in ((self.k_cache, "k_cache"), (self.v_cache, "v_cache")):
            _need(t, n, dtype)
        _need(self.len, "len", torch.int32)
        self.pyr = torch.zeros((S, H_kv, R, d), dtype=torch.float32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.sel = torch.empty((S, H_kv, K), dtype=torch.int32, device=dev)
        self.out = torch.empty((S, H_q, d), dtype=dtype, device=dev)
        self.lse = torch.empty((S, H_q), dtype=torch.float32, device=dev)
        ws = int(_lib.lib().pisa_decode_workspace_bytes(ctypes.byref(self.cfg)))
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)

    def init(self):
        """Builds each sequence's pyramid over its first len[s] cached tokens."""
        _lib.call("pisa_decode_init", ctypes.byref(self.cfg), _p(self.k_cache), _p(self.pyr), _p(self.len),
                  _stream(self.pyr))

    def _check_new(self, q_new=None, k_new=None, v_new=None):
        """Raises unless the step's tensors are [S, H_q, d] (q) and [S, H_kv, d] (k, v) in the cache dtype."""
        for t, name, H in ((q_new, "q_new", self.H_q), (k_new, "k_new", self.H_kv), (v_new, "v_new", self.H_kv)):
            if t is not None:
                _need(t, name, self.dtype, (self.S, H, self.d))

    def append(self, k_new, v_new):
        self._check_new(k_new=k_new, v_new=v_new)
        _lib.call("pisa_decode_append", ctypes.byref(self.cfg), _p(k_new), _p(v_new), _p(self.k_cache),
                  _p(self.v_cache), _p(self.pyr), _p(self.len), _p(self.status), _stream(self.pyr))

    def select(self, q_new):
        self._check_new(q_new=q_new)
        _lib.call("pisa_decode_select", ctypes.byref(self.cfg), _p(q_new), _p(self.k_cache), _p(self.pyr),
                  _p(self.len), _p(self.sel), _stream(self.pyr))
        return self.sel

    def attend(self, q_new, sel=None):
        self._check_new(q_new=q_new)
        s = self.sel if sel is None else sel
        _need(s, "sel", torch.int32, (self.S, self.H_kv, self.K))
        _lib.call("pisa_decode_attn", ctypes.byref(self.cfg), _p(q_new), _p(self.k_cache), _p(self.v_cache),
                  _p(self.len), _p(s), _p(self.out), _p(self.lse), _p(self.workspace), _stream(self.pyr))
        return self.out

    def step(self, q_new, k_new, v_new, keep_sel: bool = True):
        """Append + select + attend for every sequence."""
        self._check_new(q_new, k_new, v_new)
        _lib.call("pisa_decode_step", ctypes.byref(self.cfg), _p(q_new), _p(k_new), _p(v_new), _p(self.k_cache),
                  _p(self.v_cache), _p(self.pyr), _p(self.len), _p(self.sel) if keep_sel else None, _p(self.out),
                  _p(self.lse), _p(self.status), _p(self.workspace), _stream(self.pyr))
        return self.out

    def level_offsets(self):
        return pyramid_geometry(self.cap, self.C)[1]


class PagedDecodeState:
    """Decode state over paged KV caches: k_pages / v_pages [num_pages, H_kv,
    C, d], one leaf block of one sequence per page, and a block table
    [S, max_pages] (int32, -1 for unassigned) mapping each sequence's leaves to
    pages. The pyramid, lengths, status word and workspace are as in
    DecodeState; capacity is max_pages * C tokens per sequence."""

    def __init__(self, *, S: int, max_pages: int, H_q: int, H_kv: int, d: int, C: int, K: int, k_pages, v_pages,
                 block_table, lens, dtype=torch.bfloat16, scale: float = 0.0):
        dev = k_pages.device
        cap = max_pages * C
        self.cfg = _lib.DecodeConfig(S, cap, H_q, H_kv, d, C, 2, K, _DT[dtype], scale)
        self.S, self.cap, self.max_pages, self.H_q, self.H_kv, self.d, self.C, self.K = S, cap, max_pages, H_q, H_kv, d, C, K
        self.dtype = dtype
        if k_pages.dim() != 4:
            raise ValueError("k_pages must be [num_pages, H_kv, C, d]")
        self.num_pages = k_pages.shape[0]
        for t, n in ((k_pages, "k_pages"), (v_pages, "v_pages")):
            _need(t, n, dtype, (self.num_pages, H_kv, C, d))
        _need(block_table, "block_table", torch.int32, (S, max_pages))
        _need(lens, "lens", torch.int32, (S,))
        self.check_block_table(block_table)
        self.k_pages, self.v_pages, self.block_table, self.len = k_pages, v_pages, block_table, lens
        R = int(_lib.lib().pisa_decode_pyramid_rows(ctypes.byref(self.cfg)))
        if R <= 0:
            raise _lib.PisaError("pisa_decode_pyramid_rows", 1)
        self.R = R
        self.pyr = torch.zeros((S, H_kv, R, d), dtype=torch.float32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.sel = torch.empty((S, H_kv, K), dtype=torch.int32, device=dev)
        self.out = torch.empty((S, H_q, d), dtype=dtype, device=dev)
        self.lse = torch.empty((S, H_q), dtype=torch.float32, device=dev)
        ws = int(_lib.lib().pisa_decode_workspace_bytes(ctypes.byref(self.cfg)))
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)

    def check_block_table(self, block_table=None):
        """Raises unless every entry is -1 or a page of the pool. The kernels
        cannot bound page indices, so call this again after editing the table
        (it reads the table back to the host, which synchronises)."""
        bt = self.block_table if block_table is None else block_table
        if bt.numel() and (int(bt.min()) < -1 or int(bt.max()) >= self.num_pages):
            raise ValueError(f"block_table entries must be -1 or pages 0..{self.num_pages - 1}")

    def init(self):
        """Builds each sequence's pyramid over its first len[s] cached tokens."""
        _lib.call("pisa_decode_init_paged", ctypes.byref(self.cfg), _p(self.k_pages), _p(self.block_table),
                  self.max_pages, _p(self.pyr), _p(self.len), _stream(self.pyr))

    def step(self, q_new, k_new, v_new, keep_sel: bool = True):
        """Append + select + attend for every sequence."""
        for t, name, H in ((q_new, "q_new", self.H_q), (k_new, "k_new", self.H_kv), (v_new, "v_new", self.H_kv)):
            _need(t, name, self.dtype, (self.S, H, self.d))
        _lib.call("pisa_decode_step_paged", ctypes.byref(self.cfg), _p(q_new), _p(k_new), _p(v_new),
                  _p(self.k_pages), _p(self.v_pages), _p(self.block_table), self.max_pages, _p(self.pyr),
                  _p(self.len), _p(self.sel) if keep_sel else None, _p(self.out), _p(self.lse), _p(self.status),
                  _p(self.workspace), _stream(self.pyr))
        return self.out


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
