"""GPU-vs-oracle parity of the decode path through the C ABI: pyramid init
over per-sequence prefixes, the per-token leaf/ancestor update, the fused
root-to-leaf selection and attention for the new token, step by step through
ragged leaves and new top levels."""
import numpy as np
import pytest
import torch

import _parity as P
import oracle as O
from hierarchical_top_block_mean_b200 import api, workloads

pytestmark = pytest.mark.gpu


def _prefix_cfg(w, n):
    return O.make_cfg(B=1, N=n, H_q=w.G_Q, H_kv=1, d=w.d, C=w.C, K=w.K, causal=True,
                      dtype_code=0 if w.dtype == "f32" else 1, Nq=1, q_t0=n - 1)


def _check_seq(w, st, s, q_new, check_attn=True):
    """Compares sequence s of the decode state with the oracle on its prefix."""
    n = int(st.len[s].item())
    kc = P.host(st.k_cache[s, :, :n])
    vc = P.host(st.v_cache[s, :, :n])
    L, offs = api.pyramid_geometry(st.cap, w.C)
    pyr_gpu = P.host(st.pyr[s]).numpy()
    exempt = mism = 0
    for h in range(w.H_kv):
        ref = O.build_pyramid(kc[h:h + 1].unsqueeze(0), w.C)[0, 0]
        Ln, on = api.pyramid_geometry(n, w.C)
        for l in range(1, Ln + 1):
            got = pyr_gpu[h, offs[l - 1]:offs[l - 1] + (on[l] - on[l - 1])]
            want = ref[on[l - 1]:on[l]]
            assert np.abs(got - want).max() <= 1e-5 + 1e-6 * np.abs(want).max(), (s, h, l)
        cfg = _prefix_cfg(w, n)
        qh = P.host(q_new[s, h * w.G_Q:(h + 1) * w.G_Q]).reshape(1, w.G_Q, 1, w.d)
        sel_ref, gap = O.select_rows(cfg, qh, kc[h:h + 1].unsqueeze(0), ref[None, None], [(0, 0, n - 1)])
        sel_gpu = P.host(st.sel[s, h]).numpy()[None]
        same = (np.sort(sel_gpu, 1) == np.sort(sel_ref, 1)).all()
        if gap[0] < P.GAP_TOL:
            exempt += 1
        elif not same:
            mism += 1
        if check_attn:
            out_ref, lse_ref = O.attn_rows(cfg, qh, kc[h:h + 1].unsqueeze(0), vc[h:h + 1].unsqueeze(0),
                                           [(0, 0, n - 1)], sel_gpu)
            got = P.host(st.out[s, h * w.G_Q:(h + 1) * w.G_Q]).float().numpy()[None]
            lse = P.host(st.lse[s, h * w.G_Q:(h + 1) * w.G_Q]).numpy()[None]
            P.check_attention(w, got, lse, out_ref, lse_ref)
    assert mism == 0, f"seq {s}: {mism} non-exempt decode selection mismatches"
    return exempt


SMALL = [
    workloads.DECODE["decode_64x128k"].with_(name="dec_small", S=3, context=700, steps=70, seed=5100),
    workloads.DECODE["decode_64x128k"].with_(name="dec_small_d64_C32", S=2, context=250, steps=40, H_q=8, H_kv=2,
                                             d=64, C=32, K=5, seed=5200),
    workloads.DECODE["decode_64x128k"].with_(name="dec_small_f32", S=2, context=60, steps=80, H_q=4, H_kv=1, d=64,
                                             C=32, K=4, dtype="f32", seed=5300),
    workloads.DECODE["decode_64x128k"].with_(name="dec_small_G8", S=2, context=500, steps=40, H_q=16, H_kv=2,
                                             seed=5400),
    workloads.DECODE["decode_64x128k"].with_(name="dec_small_G1", S=2, context=420, steps=30, H_q=4, H_kv=4,
                                             K=8, seed=5500),
    workloads.DECODE["decode_64x128k"].with_(name="dec_small_G2_d64", S=3, context=200, steps=30, H_q=8, H_kv=4,
                                             d=64, C=32, K=3, seed=5600),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("fused", [True, False], ids=["step", "unfused"])
def test_decode_parity_small(w, fused):
    dev = torch.device("cuda")
    kc, vc, lens = workloads.decode_cache(w, device=dev)
    # Ragged starting lengths per sequence.
    lens -= torch.arange(w.S, device=dev, dtype=torch.int32) * 37
    st = api.DecodeState(S=w.S, cap=w.cap, H_q=w.H_q, H_kv=w.H_kv, d=w.d, C=w.C, K=w.K, dtype=w.torch_dtype,
                         device=dev, k_cache=kc, v_cache=vc, lens=lens)
    st.init()
    for step in range(w.steps):
        q, k, v = workloads.decode_step_inputs(w, step, device=dev)
        if fused:
            st.step(q, k, v)
        else:
            st.append(k, v)
            st.select(q)
            st.attend(q)
        torch.cuda.synchronize()
        if step in (0, 1, 2, 5, w.steps // 2, w.steps - 1) or step % 16 == 0:
            for s in range(w.S):
                _check_seq(w, st, s, q)
    assert int(st.status.item()) == 0


def test_decode_capacity_flag():
    w = SMALL[0].with_(S=2, context=100, steps=2)
    dev = torch.device("cuda")
    kc, vc, lens = workloads.decode_cache(w, device=dev)
    st = api.DecodeState(S=w.S, cap=w.cap, H_q=w.H_q, H_kv=w.H_kv, d=w.d, C=w.C, K=w.K, dtype=w.torch_dtype,
                         device=dev, k_cache=kc, v_cache=vc, lens=lens)
    st.init()
    for step in range(3):
        q, k, v = workloads.decode_step_inputs(w, step, device=dev)
        st.step(q, k, v)
    torch.cuda.synchronize()
    assert int(st.status.item()) == 4  # PISA_ERR_CAPACITY, sequences stopped at cap
    assert st.len.tolist() == [w.cap, w.cap]


@pytest.mark.slow
def test_decode_parity_full_size_sampled():
    w = workloads.DECODE["decode_64x128k"]
    dev = torch.device("cuda")
    kc, vc, lens = workloads.decode_cache(w, device=dev)
    st = api.DecodeState(S=w.S, cap=w.cap, H_q=w.H_q, H_kv=w.H_kv, d=w.d, C=w.C, K=w.K, dtype=w.torch_dtype,
                         device=dev, k_cache=kc, v_cache=vc, lens=lens)
    st.init()
    check_steps = {0, 1, 63, 255}
    seqs = [0, 17, 42, 63]
    for step in range(w.steps):
        q, k, v = workloads.decode_step_inputs(w, step, device=dev)
        st.step(q, k, v)
        if step in check_steps:
            torch.cuda.synchronize()
            for s in seqs:
                _check_seq(w, st, s, q)
    assert int(st.status.item()) == 0
