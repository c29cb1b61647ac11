"""The Python binding's argument checks, on CPU. The kernels trust every size
they are given, so a user buffer of the wrong shape, dtype or layout must be
refused before the C call. The device check, the stream lookup and the C call
itself are stubbed: CPU tensors stand in for device tensors, and each entry
point records its call instead of launching. Valid shapes (those the GPU
tests use) must reach the C call; each wrong buffer must raise ValueError
without reaching it."""
import pytest
import torch

from hierarchical_top_block_mean_b200 import _lib, api

B, N, H_q, H_kv, d, C, K = 1, 300, 8, 2, 64, 32, 4
bf = torch.bfloat16


@pytest.fixture
def calls(monkeypatch):
    rec = []
    monkeypatch.setattr(api, "_on_cuda", lambda t, name: None)
    monkeypatch.setattr(api, "_stream", lambda t: None)
    monkeypatch.setattr(api, "_p", lambda t: None)
    monkeypatch.setattr(_lib, "call", lambda name, *a: rec.append(name))
    return rec


def _qkv(n_q=N):
    return (torch.zeros(B, H_q, n_q, d, dtype=bf), torch.zeros(B, H_kv, N, d, dtype=bf),
            torch.zeros(B, H_kv, N, d, dtype=bf))


def _R():
    return api.pyramid_rows(N, C)


def test_valid_calls_reach_the_library(calls):
    q, k, v = _qkv()
    pyr = api.build_pyramid(k, C=C)
    assert tuple(pyr.shape) == (B, H_kv, _R(), d)
    sel = api.select(q, k, pyr, C=C, K=K, causal=True, score=torch.zeros(B, H_kv, N, K))
    api.select_flat(q, pyr, C=C, K=K, causal=True, H_kv=H_kv, out=torch.zeros(B, H_kv, N, K, dtype=torch.int32))
    api.select_exact(q, k, C=C, K=K, causal=True)
    out, lse = api.sparse_attn_fwd(q, k, v, sel, C=C, causal=True)
    api.sparse_attn_bwd(q, k, v, sel, out, lse, torch.zeros_like(q), C=C, causal=True)
    qs = q[:, :, 100:250].contiguous()
    ssel = api.select_span(qs, k, pyr, q0=100, C=C, K=K, causal=True)
    api.sparse_attn_fwd_span(qs, k, v, ssel, q0=100, C=C, causal=True)
    pr = api.Problem.of(q, k, C=C, K=K, causal=True)
    api.Prefill(pr, "cpu")(q, k, v)
    api.PrefillShard(pr, 100, 150, "cpu")(qs, k, v)
    assert calls == ["pisa_build_pyramid", "pisa_select", "pisa_select_flat", "pisa_select_exact",
                     "pisa_sparse_attn_fwd", "pisa_sparse_attn_bwd", "pisa_select_span", "pisa_sparse_attn_fwd_span",
                     "pisa_build_pyramid", "pisa_select", "pisa_sparse_attn_fwd",
                     "pisa_build_pyramid", "pisa_select_span", "pisa_sparse_attn_fwd_span"]


def _refused(calls, fn, *a, **kw):
    n = len(calls)
    with pytest.raises(ValueError):
        fn(*a, **kw)
    assert len(calls) == n, "a refused call reached the library"


def test_wrong_buffers_are_refused(calls):
    q, k, v = _qkv()
    R = _R()
    pyr = torch.zeros(B, H_kv, R, d)
    sel = torch.zeros(B, H_kv, N, K, dtype=torch.int32)
    i32 = torch.int32
    _refused(calls, api.build_pyramid, k, C=C, out=torch.zeros(B, H_kv, R - 1, d))
    _refused(calls, api.select, q, k, pyr[:, :, :-1].contiguous(), C=C, K=K, causal=True)
    _refused(calls, api.select, q, k, pyr.double(), C=C, K=K, causal=True)
    _refused(calls, api.select, q, k, pyr, C=C, K=K, causal=True, out=torch.zeros(B, H_kv, N, K - 1, dtype=i32))
    _refused(calls, api.select, q, k, pyr, C=C, K=K, causal=True, score=torch.zeros(B, H_kv, N - 1, K))
    _refused(calls, api.select_flat, q, pyr, C=C, K=K, causal=True, H_kv=H_kv,
             out=torch.zeros(B, H_kv, N, K, dtype=torch.int64))
    _refused(calls, api.select_exact, q, k, C=C, K=K, causal=True, out=torch.zeros(B, H_kv, N - 1, K, dtype=i32))
    _refused(calls, api.sparse_attn_fwd, q, k, v[:, :, :-1].contiguous(), sel, C=C, causal=True)
    _refused(calls, api.sparse_attn_fwd, q, k, v, sel[:, :, :-1].contiguous(), C=C, causal=True)
    _refused(calls, api.sparse_attn_fwd, q, k, v, sel, C=C, causal=True, out=torch.zeros_like(q).float())
    _refused(calls, api.sparse_attn_fwd, q, k, v, sel, C=C, causal=True, lse=torch.zeros(B, H_q, N - 1))
    _refused(calls, api.sparse_attn_fwd, q, k, v, sel.transpose(2, 3), C=C, causal=True)  # wrong shape
    _refused(calls, api.sparse_attn_fwd, q, k, v, sel.permute(0, 1, 2, 3)[:, :, ::2], C=C, causal=True)
    out, lse = torch.zeros_like(q), torch.zeros(B, H_q, N)
    _refused(calls, api.sparse_attn_bwd, q, k, v, sel, out, lse[:, :, :-1].contiguous(), q, C=C, causal=True)
    _refused(calls, api.sparse_attn_bwd, q, k, v, sel, out[:, :, :-1].contiguous(), lse, q, C=C, causal=True)
    qs = q[:, :, 100:250].contiguous()
    _refused(calls, api.select_span, qs, k, pyr, q0=100, C=C, K=K, causal=True,
             out=torch.zeros(B, H_kv, N, K, dtype=i32))  # whole-sequence rows, not the shard's
    _refused(calls, api.sparse_attn_fwd_span, qs, k, v, sel, q0=100, C=C, causal=True)
    pr = api.Problem.of(q, k, C=C, K=K, causal=True)
    _refused(calls, api.Prefill(pr, "cpu"), q[:, :, :-1].contiguous(), k, v)
    _refused(calls, api.PrefillShard(pr, 100, 150, "cpu"), q, k, v)


def test_decode_state_checks_step_tensors(calls):
    S, cap, Hq, Hkv = 3, 500, 8, 2
    st = api.DecodeState(S=S, cap=cap, H_q=Hq, H_kv=Hkv, d=d, C=C, K=K, device="cpu")
    qn, kn, vn = torch.zeros(S, Hq, d, dtype=bf), torch.zeros(S, Hkv, d, dtype=bf), torch.zeros(S, Hkv, d, dtype=bf)
    st.step(qn, kn, vn)
    st.append(kn, vn)
    st.select(qn)
    st.attend(qn)
    assert calls == ["pisa_decode_step", "pisa_decode_append", "pisa_decode_select", "pisa_decode_attn"]
    _refused(calls, st.step, qn[:, :Hkv].contiguous(), kn, vn)
    _refused(calls, st.step, qn, kn.float(), vn)
    _refused(calls, st.append, kn, vn[:-1].contiguous())
    _refused(calls, st.attend, qn, torch.zeros(S, Hkv, K + 1, dtype=torch.int32))
    pages = torch.zeros(4 * S, Hkv, C, d, dtype=bf)
    bt = torch.zeros(S, 4, dtype=torch.int32)
    ps = api.PagedDecodeState(S=S, max_pages=4, H_q=Hq, H_kv=Hkv, d=d, C=C, K=K, k_pages=pages, v_pages=pages,
                              block_table=bt, lens=torch.zeros(S, dtype=torch.int32))
    ps.step(qn, kn, vn)
    assert calls[-1] == "pisa_decode_step_paged"
    _refused(calls, ps.step, qn, kn, vn[:, :, :-1].contiguous())


def test_paged_state_refuses_out_of_pool_pages(calls):
    S, Hq, Hkv, P = 2, 8, 2, 5
    pages = torch.zeros(P, Hkv, C, d, dtype=bf)
    lens = torch.zeros(S, dtype=torch.int32)

    def make(bt, kp=pages):
        return api.PagedDecodeState(S=S, max_pages=3, H_q=Hq, H_kv=Hkv, d=d, C=C, K=K, k_pages=kp, v_pages=kp,
                                    block_table=bt, lens=lens)

    ok = make(torch.tensor([[0, 1, -1], [2, 3, 4]], dtype=torch.int32))
    for bad in ([[0, 1, 5], [2, 3, 4]], [[0, -2, 1], [2, 3, 4]]):
        with pytest.raises(ValueError):
            make(torch.tensor(bad, dtype=torch.int32))
    with pytest.raises(ValueError):
        make(torch.zeros(S, 2, dtype=torch.int32))  # not [S, max_pages]
    with pytest.raises(ValueError):
        make(torch.zeros(S, 3, dtype=torch.int32), kp=torch.zeros(P, Hkv, C // 2, d, dtype=bf))
    ok.block_table[1, 2] = P  # an edit after construction is caught by the explicit check
    with pytest.raises(ValueError):
        ok.check_block_table()
    assert calls == []


def test_tensor_on_another_device_is_refused(monkeypatch):
    # The library launches on the current device; a tensor on another GPU
    # (or tensors of one call spread over GPUs) must be refused before the C
    # call. The current device is stubbed to cuda:0.
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    api._check_device_index(0, "q")
    with pytest.raises(ValueError, match="cuda:1"):
        api._check_device_index(1, "k")
