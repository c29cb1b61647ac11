"""Host logic of sequence-parallel prefill on CPU: the shard arithmetic, and
the all-gather that assembles every rank's key and value slices into the
full [B, H, N, d] tensors, run as two gloo ranks."""
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


@pytest.mark.parametrize("shape", [(1, 2, 64, 8), (2, 3, 10, 4)])
def test_gather_sequence_two_ranks(shape):
    ctx = mp.get_context("spawn")
    errq = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_rank, args=(r, 2, port, shape, errq)) for r in range(2)]
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
