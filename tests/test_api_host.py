"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/pisa.h declares, its integer pyramid geometry matches
the oracle bit for bit, and argument validation rejects bad calls before
anything is enqueued."""
import ctypes
import os
import re

import numpy as np
import pytest

from hierarchical_top_block_mean_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "pisa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(pisa_[a-z_0-9]+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    lib = _lib.lib()
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES)


def test_status_strings_and_version():
    lib = _lib.lib()
    for code, name in _lib.STATUS_NAMES.items():
        assert lib.pisa_status_string(code).decode() == name
    assert lib.pisa_version() >= 100


@pytest.mark.parametrize("N,C", [(1, 32), (5, 32), (1024, 32), (1000, 64), (16384, 64), (131328, 64),
                                 (262144, 64), (77777, 32)])
def test_geometry_matches_oracle(oracle, N, C):
    from hierarchical_top_block_mean_b200 import pyramid_geometry, pyramid_rows
    L, offs = pyramid_geometry(N, C)
    sizes, ooffs = oracle.geometry(N, C)
    assert L == len(sizes) - 1
    assert offs == list(ooffs)
    assert pyramid_rows(N, C) == ooffs[-1]


def _cfg(**kw):
    base = dict(B=1, N=256, H_q=4, H_kv=1, d=64, C=32, g=2, K=4, q_tile=4, causal=1, dtype=1, scale=0.0)
    base.update(kw)
    return _lib.Config(*[base[f] for f, _ in _lib.Config._fields_])


@pytest.mark.parametrize("kw,code", [
    (dict(N=1 << 27), 2), (dict(B=64, N=1 << 22, H_q=8), 2),
    (dict(N=0), 1), (dict(B=0), 1), (dict(H_q=6, H_kv=4), 1), (dict(dtype=7), 1), (dict(causal=2), 1),
    (dict(g=3), 2), (dict(C=16), 2), (dict(d=96), 2), (dict(K=17), 2), (dict(q_tile=8), 2),
    (dict(H_q=12, H_kv=1), 2),
])
def test_invalid_configs_rejected_before_launch(kw, code):
    lib = _lib.lib()
    before = lib.pisa_launch_count()
    dummy = ctypes.c_void_p(256)
    cfg = _cfg(**kw)
    assert lib.pisa_build_pyramid(ctypes.byref(cfg), dummy, dummy, None) == code
    assert lib.pisa_select(ctypes.byref(cfg), dummy, dummy, dummy, dummy, None, dummy, 1 << 30, None) == code
    assert lib.pisa_select_flat(ctypes.byref(cfg), dummy, dummy, dummy, dummy, 1 << 30, None) == code
    assert lib.pisa_sparse_attn_fwd(ctypes.byref(cfg), dummy, dummy, dummy, dummy, dummy, None, None, 0, None) == code
    assert lib.pisa_select_exact(ctypes.byref(cfg), dummy, dummy, dummy, None) == code
    assert lib.pisa_sparse_attn_bwd(ctypes.byref(cfg), dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy,
                                    dummy, dummy, 1 << 30, None) == code
    assert lib.pisa_select_workspace_bytes(ctypes.byref(cfg)) == 0
    assert lib.pisa_select_flat_workspace_bytes(ctypes.byref(cfg)) == 0
    assert lib.pisa_attn_bwd_workspace_bytes(ctypes.byref(cfg)) == 0
    assert lib.pisa_launch_count() == before


def test_null_and_misaligned_pointers_rejected():
    lib = _lib.lib()
    cfg = _cfg()
    ok = ctypes.c_void_p(256)
    bad = ctypes.c_void_p(258)
    assert lib.pisa_build_pyramid(ctypes.byref(cfg), None, ok, None) == 1
    assert lib.pisa_build_pyramid(ctypes.byref(cfg), bad, ok, None) == 1
    assert lib.pisa_sparse_attn_fwd(ctypes.byref(cfg), ok, ok, ok, None, ok, None, None, 0, None) == 1
    assert lib.pisa_select(ctypes.byref(cfg), None, ok, ok, ok, None, ok, 1 << 30, None) == 1
    assert lib.pisa_build_pyramid(None, ok, ok, None) == 1


def test_select_workspace_too_small_rejected():
    lib = _lib.lib()
    cfg = _cfg(dtype=1)
    need = lib.pisa_select_workspace_bytes(ctypes.byref(cfg))
    assert need > 0
    ok = ctypes.c_void_p(256)
    assert lib.pisa_select(ctypes.byref(cfg), ok, ok, ok, ok, None, ok, need - 1, None) == 3
    assert lib.pisa_select(ctypes.byref(cfg), ok, ok, ok, ok, None, None, need, None) == 3


def test_decode_validation():
    lib = _lib.lib()
    dc = _lib.DecodeConfig(2, 300, 8, 2, 64, 32, 2, 4, 1, 0.0)
    R = lib.pisa_decode_pyramid_rows(ctypes.byref(dc))
    assert R == lib.pisa_pyramid_rows(300, 32)
    bad = _lib.DecodeConfig(2, 0, 8, 2, 64, 32, 2, 4, 1, 0.0)
    assert lib.pisa_decode_pyramid_rows(ctypes.byref(bad)) == 0
    ok = ctypes.c_void_p(256)
    assert lib.pisa_decode_append(ctypes.byref(dc), ok, ok, ok, ok, ok, ok, None, None) == 1  # status word required
    assert lib.pisa_decode_step(ctypes.byref(bad), ok, ok, ok, ok, ok, ok, ok, None, ok, None, ok, ok, None) == 1
    assert lib.pisa_decode_workspace_bytes(ctypes.byref(bad)) == 0


def test_decode_workspace_size():
    """The fused path keeps fp32 logits of 2K leaf blocks of C keys for the G_Q
    heads of every (sequence, kv head); the fp32 fallback needs none."""
    lib = _lib.lib()
    S, cap, H_q, H_kv, d, C, K = 3, 4096, 16, 4, 128, 64, 16
    bf = _lib.DecodeConfig(S, cap, H_q, H_kv, d, C, 2, K, 1, 0.0)
    assert lib.pisa_decode_workspace_bytes(ctypes.byref(bf)) == S * H_kv * 2 * K * C * (H_q // H_kv) * 4
    f32 = _lib.DecodeConfig(S, cap, H_q, H_kv, d, C, 2, K, 0, 0.0)
    assert lib.pisa_decode_workspace_bytes(ctypes.byref(f32)) == 0
    ok = ctypes.c_void_p(256)
    # A needed workspace that is missing is refused before anything is enqueued.
    assert lib.pisa_decode_step(ctypes.byref(bf), ok, ok, ok, ok, ok, ok, ok, None, ok, None, ok, None, None) == 3
    assert lib.pisa_decode_attn(ctypes.byref(bf), ok, ok, ok, ok, ok, ok, None, None, None) == 3


def test_query_span_validation():
    """A query shard must lie inside the sequence; a bad span is refused before
    anything is enqueued, and a whole-sequence span is the plain call."""
    lib = _lib.lib()
    before = lib.pisa_launch_count()
    cfg = _cfg(N=1000, dtype=1)
    ok = ctypes.c_void_p(256)
    whole = _lib.QuerySpan(0, 1000)
    assert lib.pisa_select_span_workspace_bytes(ctypes.byref(cfg), ctypes.byref(whole)) == \
        lib.pisa_select_workspace_bytes(ctypes.byref(cfg))
    part = _lib.QuerySpan(500, 250)
    need = lib.pisa_select_span_workspace_bytes(ctypes.byref(cfg), ctypes.byref(part))
    assert 0 < need < lib.pisa_select_workspace_bytes(ctypes.byref(cfg))
    for q0, n_q in ((-1, 10), (0, 0), (990, 11), (1000, 1), (0, 1001)):
        sp = _lib.QuerySpan(q0, n_q)
        assert lib.pisa_select_span_workspace_bytes(ctypes.byref(cfg), ctypes.byref(sp)) == 0
        assert lib.pisa_select_span(ctypes.byref(cfg), ctypes.byref(sp), ok, ok, ok, ok, None, ok, 1 << 30,
                                    None) == 1
        assert lib.pisa_sparse_attn_fwd_span(ctypes.byref(cfg), ctypes.byref(sp), ok, ok, ok, ok, ok, None,
                                             None, 0, None) == 1
        assert lib.pisa_attn_fwd_span_workspace_bytes(ctypes.byref(cfg), ctypes.byref(sp)) == 0
    assert lib.pisa_select_span(ctypes.byref(cfg), None, ok, ok, ok, ok, None, ok, 1 << 30, None) == 1
    assert lib.pisa_sparse_attn_fwd_span(ctypes.byref(cfg), None, ok, ok, ok, ok, ok, None, None, 0, None) == 1
    assert lib.pisa_select_span(ctypes.byref(cfg), ctypes.byref(part), ok, ok, ok, ok, None, ok, need - 1, None) == 3
    assert lib.pisa_launch_count() == before


def test_header_compiles_as_c99_and_links(tmp_path):
    """The boundary is a C ABI: a plain C99 program includes pisa.h, links the
    library and runs its host-only calls (no GPU needed)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(_lib.LIB_PATH)
    exe = str(tmp_path / "abi_check")
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_check.c"), "-L", lib_dir, "-lpisa_b200",
                    "-Wl,-rpath," + lib_dir, "-o", exe], check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "FAIL" not in r.stdout and r.stdout.count("ok ") == 15, r.stdout


def test_flat_workspace_sized_and_checked_before_launch():
    # bf16 with d = 128 takes the tensor-core flat selector, whose hi/lo
    # operand planes live in the caller's workspace: 2 x (B H_kv N + B H_kv M_1)
    # rows of 128 bf16, each plane 256-byte aligned. Too small a workspace is
    # refused before anything is enqueued; other shapes need none.
    lib = _lib.lib()
    cfg = _cfg(N=1000, H_q=8, H_kv=2, d=128, C=64)
    need = lib.pisa_select_flat_workspace_bytes(ctypes.byref(cfg))
    rows_q, rows_k = 2 * 1000, 2 * 16
    al = lambda x: (x + 255) // 256 * 256
    assert need == 2 * al(rows_q * 256) + 2 * al(rows_k * 256)
    before = lib.pisa_launch_count()
    dummy = ctypes.c_void_p(256)
    assert lib.pisa_select_flat(ctypes.byref(cfg), dummy, dummy, dummy, dummy, need - 1, None) == 3
    assert lib.pisa_select_flat(ctypes.byref(cfg), dummy, dummy, dummy, None, need, None) == 3
    assert lib.pisa_launch_count() == before
    assert lib.pisa_select_flat_workspace_bytes(ctypes.byref(_cfg(N=1000, d=64, C=32))) == 0


def test_attention_workspace_sized_and_checked_before_launch():
    # The bucketed attention (bf16, d = 128, C = 64, G_Q in {4, 8}) keeps a
    # partial softmax state per (query, selected block, head) in the caller's
    # workspace: at least rows * K * G_Q * (256 + 8) bytes. A shard needs
    # scratch for its own rows only. Too small a workspace is refused before
    # anything is enqueued; other shapes report 0 and stream rows without one.
    lib = _lib.lib()
    cfg = _cfg(N=1000, H_q=8, H_kv=2, d=128, C=64, K=16)
    need = lib.pisa_attn_fwd_workspace_bytes(ctypes.byref(cfg))
    assert need >= 2 * 1000 * 16 * 4 * 264
    half = _lib.QuerySpan(500, 500)
    assert 0 < lib.pisa_attn_fwd_span_workspace_bytes(ctypes.byref(cfg), ctypes.byref(half)) < need
    before = lib.pisa_launch_count()
    ok = ctypes.c_void_p(1024)
    assert lib.pisa_sparse_attn_fwd(ctypes.byref(cfg), ok, ok, ok, ok, ok, None, ok, need - 1, None) == 3
    assert lib.pisa_launch_count() == before
    for kw in (dict(d=64, C=32), dict(H_q=2, H_kv=2, d=128, C=64), dict(d=128, C=32, H_q=8, H_kv=2),
               dict(dtype=0, d=128, C=64, H_q=8, H_kv=2)):
        assert lib.pisa_attn_fwd_workspace_bytes(ctypes.byref(_cfg(N=1000, **kw))) == 0
