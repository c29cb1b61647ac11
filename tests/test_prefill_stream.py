"""PrefillStream: prefill steps fed from pinned host memory with the copies
overlapped with compute on two copy streams and double-buffered slots. Each
step's output, read back into host memory, must equal a plain Prefill of
the same batch bit for bit. Five batches of different inputs are submitted
back to back, so every slot is reused while the other is busy, and a wrong
event order would hand a step another batch's inputs or output."""
import pytest
import torch

from hierarchical_top_block_mean_b200 import api, workloads

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("depth", [1, 2, 3])
def test_stream_outputs_equal_plain_prefill(depth):
    dev = torch.device("cuda")
    base = workloads.PREFILL["needle_256k"].with_(name="stream_4k", N=4096, n_needles=8)
    batches = [workloads.prefill_inputs(base.with_(seed=9700 + i), device=dev) for i in range(5)]
    pr = api.Problem.of(batches[0]["q"], batches[0]["k"], C=base.C, K=base.K, causal=base.causal)
    ref = api.Prefill(pr, dev)
    want = []
    for x in batches:
        ref(x["q"], x["k"], x["v"])
        want.append(ref.out.cpu())
    host = [tuple(x[n].cpu().pin_memory() for n in ("q", "k", "v")) for x in batches]
    outs = [torch.empty(want[0].shape, dtype=want[0].dtype).pin_memory() for _ in batches]
    ps = api.PrefillStream(pr, dev, depth=depth)
    for (hq, hk, hv), ho in zip(host, outs):
        ps.submit(hq, hk, hv, ho)
    ps.synchronize()
    for i, (got, exp) in enumerate(zip(outs, want)):
        assert torch.equal(got, exp), f"depth {depth}: step {i} output differs from a plain prefill"


def test_stream_rejects_unpinned_or_misshaped_host_tensors():
    dev = torch.device("cuda")
    w = workloads.PREFILL["needle_256k"].with_(name="stream_small", N=512, n_needles=0, structure="iid")
    x = workloads.prefill_inputs(w, device=dev)
    pr = api.Problem.of(x["q"], x["k"], C=w.C, K=w.K, causal=w.causal)
    ps = api.PrefillStream(pr, dev)
    hq, hk, hv = (x[n].cpu().pin_memory() for n in ("q", "k", "v"))
    ho = torch.empty(x["q"].shape, dtype=x["q"].dtype).pin_memory()
    with pytest.raises(ValueError):
        ps.submit(x["q"].cpu(), hk, hv, ho)  # pageable
    with pytest.raises(ValueError):
        ps.submit(hq, hk, hv, ho[:, :, :-1])  # wrong shape
    with pytest.raises(ValueError):
        ps.submit(x["q"], hk, hv, ho)  # device tensor
    ps.submit(hq, hk, hv, ho)
    ps.synchronize()
