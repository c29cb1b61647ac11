"""Sequence-parallel prefill: one sequence's tokens split by position over
the ranks of a process group, one process per GPU.

Rank r holds tokens [r n, (r + 1) n) of q, k and v (n = N / P for P ranks).
A query row's selection and attention read all earlier keys, so the one
exchange is an all-gather of the key and value slices into full [B, H_kv, N,
d] copies on every rank. Each rank then builds the whole pyramid (one read of
the gathered keys), and selects and attends for its own query rows through
the query-span entry points of the C ABI. Rows are independent (§TopK,
§BSA), so the ranks' outputs are bit-for-bit the rows of a one-GPU run.

The gathers run on the communicator's stream. The values' gather overlaps
the pyramid and the selection, which need only the keys. Each (batch, kv
head) plane of the full tensors is contiguous, and rank r's slice is its
r-th chunk, so one all-gather per plane writes the slices in place with no
reordering copy.

The exchange goes through torch.distributed (NCCL over NVLink on GPUs, gloo
on CPU for host-side tests). The kernels read only this GPU's memory.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from .api import PrefillShard, Problem, _need


def shard_span(N: int, world: int, rank: int) -> tuple[int, int]:
    """(q0, n) of rank's slice: equal slices of N / world tokens, in rank order."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if N % world != 0:
        raise ValueError(f"N = {N} must split into {world} equal slices")
    n = N // world
    return rank * n, n


def gather_sequence(x_local: torch.Tensor, x_full: torch.Tensor, group=None, async_op: bool = True):
    """All-gathers rank slices [B, H, n, d] into x_full [B, H, world n, d]
    along the token axis, one collective per (batch, head) plane. Returns the
    list of work handles (async_op) or None."""
    world = dist.get_world_size(group)
    B, H, n, d = x_local.shape
    if tuple(x_full.shape) != (B, H, world * n, d):
        raise ValueError(f"x_full {tuple(x_full.shape)} is not [B, H, {world} x {n}, d]")
    if not (x_local.is_contiguous() and x_full.is_contiguous()):
        raise ValueError("gather_sequence needs contiguous tensors")
    works = []
    for b in range(B):
        for h in range(H):
            w = dist.all_gather_into_tensor(x_full[b, h], x_local[b, h], group=group, async_op=async_op)
            if async_op:
                works.append(w)
    return works if async_op else None


class SeqParallelPrefill:
    """Prefill of one sequence of N tokens split over the ranks of `group`.

    Holds the full key and value buffers and this rank's shard (pyramid,
    selection, output and lse rows, workspace), all allocated once. Call it
    with this rank's slices q, k, v [B, H, n, d]. It returns (out [B, H_q, n,
    d], lse [B, H_q, n], sel [B, H_kv, n, K]) for query positions [q0, q0 + n).

    `shard` replaces the per-rank compute; by default it is a PrefillShard
    (the CUDA kernels) for this rank's span. Anything with pyramid(k),
    select(q, k), attend(q, k, v) and out, lse, sel attributes will do."""

    def __init__(self, pr: Problem, group=None, device="cuda", shard=None):
        self.pr, self.group = pr, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.q0, self.n = shard_span(pr.N, self.world, self.rank)
        dev = torch.device(device)
        if dev.type == "cuda" and shard is None and dev.index is not None:
            torch.cuda.set_device(dev)  # the library launches on the current device
        self._kernels = shard is None  # the default shard runs the library's CUDA kernels
        self.shard = PrefillShard(pr, self.q0, self.n, dev) if shard is None else shard
        self.k_full = torch.empty((pr.B, pr.H_kv, pr.N, pr.d), dtype=pr.dtype, device=dev)
        self.v_full = torch.empty_like(self.k_full)

    def _check(self, q, k, v):
        pr = self.pr
        for t, name, H in ((q, "q", pr.H_q), (k, "k", pr.H_kv), (v, "v", pr.H_kv)):
            if self._kernels:
                _need(t, name, pr.dtype)
            elif t.dtype != pr.dtype or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous {pr.dtype} tensor")
            if tuple(t.shape) != (pr.B, H, self.n, pr.d):
                raise ValueError(f"{name} {tuple(t.shape)} is not this rank's slice [{pr.B}, {H}, {self.n}, {pr.d}]")

    def __call__(self, q, k, v):
        self._check(q, k, v)
        wk = gather_sequence(k, self.k_full, self.group)
        wv = gather_sequence(v, self.v_full, self.group)
        for w in wk:
            w.wait()  # the current stream waits for the keys' gather
        self.shard.pyramid(self.k_full)
        self.shard.select(q, self.k_full)
        for w in wv:
            w.wait()
        self.shard.attend(q, self.k_full, self.v_full)
        return self.shard.out, self.shard.lse, self.shard.sel
