"""Host logic of sequence-parallel prefill on CPU, run as gloo ranks (two, and four for the gather):
the shard arithmetic; the all-gather that assembles every rank's key and
value slices into the full [B, H, N, d] tensors; and the driver's order of
steps, with a recording stand-in for the CUDA shard. The pyramid must see
the gathered keys, the selection this rank's queries and the keys, and the
attention the gathered values."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from hierarchical_top_block_mean_b200 import seqpar


def test_shard_span():
    assert [seqpar.shard_span(1024, 4, r) for r in range(4)] == [(0, 256), (256, 256), (512, 256), (768, 256)]
    assert seqpar.shard_span(7, 1, 0) == (0, 7)
    with pytest.raises(ValueError):
        seqpar.shard_span(1000, 3, 0)
    with pytest.raises(ValueError):
        seqpar.shard_span(1024, 4, 4)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gather_rank(rank, world, port, shape, errq):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        dist.init_process_group("gloo", rank=rank, world_size=world)
        B, H, N, d = shape
        g = torch.Generator().manual_seed(123)
        full = torch.randn(shape, generator=g)          # the same on every rank
        q0, n = seqpar.shard_span(N, world, rank)
        local = full[:, :, q0:q0 + n].contiguous()
        out = torch.full(shape, float("nan"))
        for w in seqpar.gather_sequence(local, out):
            w.wait()
        assert torch.equal(out, full), f"rank {rank}: gathered tensor differs"
        out2 = torch.full(shape, float("nan"))
        assert seqpar.gather_sequence(local, out2, async_op=False) is None
        assert torch.equal(out2, full)
        with pytest.raises(ValueError):
            seqpar.gather_sequence(local, torch.empty(B, H, N + 1, d))
        dist.barrier()
        dist.destroy_process_group()
    except BaseException as e:  # report to the parent instead of hanging it
        errq.put(f"rank {rank}: {type(e).__name__}: {e}")
        raise


@pytest.mark.parametrize("world,shape", [(2, (1, 2, 64, 8)), (2, (2, 3, 10, 4)), (4, (1, 3, 96, 4))])
def test_gather_sequence_ranks(world, shape):
    ctx = mp.get_context("spawn")
    errq = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_rank, args=(r, world, port, shape, errq)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    errs = []
    while not errq.empty():
        errs.append(errq.get())
    assert not errs, errs
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]


class _RecordingShard:
    """Stands in for the CUDA shard: records what each step sees."""

    def __init__(self, pr, q0, n):
        self.q0, self.n = q0, n
        self.calls = []
        self.out = torch.zeros(pr.B, pr.H_q, n, pr.d)
        self.lse = torch.zeros(pr.B, pr.H_q, n)
        self.sel = torch.zeros(pr.B, pr.H_kv, n, pr.K, dtype=torch.int32)

    def pyramid(self, k):
        self.calls.append(("pyramid", k.clone()))

    def select(self, q, k):
        self.calls.append(("select", q.clone(), k.clone()))

    def attend(self, q, k, v):
        self.calls.append(("attend", q.clone(), k.clone(), v.clone()))


def _driver_rank(rank, world, port, errq):
    try:
        from hierarchical_top_block_mean_b200 import api
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        dist.init_process_group("gloo", rank=rank, world_size=world)
        pr = api.Problem(B=1, N=96, H_q=4, H_kv=2, d=8, C=32, K=2, causal=True, dtype=torch.float32)
        g = torch.Generator().manual_seed(7)
        q, k, v = (torch.randn(pr.B, H, pr.N, pr.d, generator=g) for H in (pr.H_q, pr.H_kv, pr.H_kv))
        q0, n = seqpar.shard_span(pr.N, world, rank)
        fake = _RecordingShard(pr, q0, n)
        sp = seqpar.SeqParallelPrefill(pr, device="cpu", shard=fake)
        assert (sp.q0, sp.n) == (q0, n) == (rank * 48, 48)
        sl = lambda x: x[:, :, q0:q0 + n].contiguous()
        out, lse, sel = sp(sl(q), sl(k), sl(v))
        assert out is fake.out and lse is fake.lse and sel is fake.sel
        names = [c[0] for c in fake.calls]
        assert names == ["pyramid", "select", "attend"], names
        # Every step sees the whole sequence's keys (and values), this rank's own queries.
        assert torch.equal(fake.calls[0][1], k)
        assert torch.equal(fake.calls[1][1], sl(q)) and torch.equal(fake.calls[1][2], k)
        assert torch.equal(fake.calls[2][2], k) and torch.equal(fake.calls[2][3], v)
        with pytest.raises(ValueError):  # another rank's slice length is refused before any collective
            sp(q, sl(k), sl(v))
        dist.barrier()
        dist.destroy_process_group()
    except BaseException as e:
        errq.put(f"rank {rank}: {type(e).__name__}: {e}")
        raise


def test_driver_two_ranks_orchestration():
    ctx = mp.get_context("spawn")
    errq = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_driver_rank, args=(r, 2, port, errq)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    errs = []
    while not errq.empty():
        errs.append(errq.get())
    assert not errs, errs
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
