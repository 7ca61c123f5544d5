"""Host-side checks of the C ABI (no GPU needed, no kernel is launched).

The library must load, export every function include/hs2.h declares, and reject
bad arguments synchronously, before anything is enqueued.
"""
import ctypes
import os
import re

import pytest

import kv_shared_b200 as hs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "hs2.h")).read()
    return sorted(set(re.findall(r"HS2_API\s+[\w\s\*]+?\b(hs2_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(hs.LIB_PATH):
        import __graft_entry__
        __graft_entry__.build()
    return hs.lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L, n), n
    assert sorted(hs.EXPORTS) == names


def test_status_strings(L):
    for code in range(7):
        assert hs.status_string(code)
    assert hs.status_string(99) == "unknown status"


def _desc(**kw):
    base = dict(batch=2, n_q=1, heads=16, head_dim=128, max_ctx=4096)
    base.update(kw)
    return hs.make_desc(**base)


def test_workspace_size_valid_and_invalid(L):
    d = _desc()
    n1 = hs.hs2_workspace_size(d, True)
    n0 = hs.hs2_workspace_size(d, False)
    assert n1 > n0 > 256
    assert hs.hs2_workspace_size(_desc(head_dim=96)) == 0           # unsupported dim
    assert hs.hs2_workspace_size(_desc(heads=8)) == 0               # tensor-core path needs 16 heads
    assert hs.hs2_workspace_size(_desc(max_ctx=0)) == 0
    assert hs.hs2_workspace_size(_desc(idx_stride=100)) == 0        # < window + budget
    f32 = _desc(heads=8, head_dim=64, q_dtype=hs.HS2_F32, kv_dtype=hs.HS2_F32, n_q=64, max_ctx=64)
    assert hs.hs2_workspace_size(f32, True) >= 256 + 64 * 64 * 4


def test_full_attn_launch_count(L):
    # host-side plan: decode contexts whose splits fit tensor memory take one launch plus
    # the selection; longer ones (1M keys: more than 148 x 4096) take three (two passes and
    # the merge of the split partials) plus the selection (one launch either way: the cluster
    # select for rows up to 393216 keys, the selection from the histograms beyond)
    assert hs.hs2_full_attn_launches(_desc(batch=32, max_ctx=131072)) == 2
    assert hs.hs2_full_attn_launches(_desc(batch=2, max_ctx=450000)) == 2
    assert hs.hs2_full_attn_launches(_desc(batch=4, max_ctx=1 << 20, kv_dtype=hs.HS2_E4M3)) == 4
    assert hs.hs2_full_attn_launches(_desc(batch=4, n_q=8192, max_ctx=65536 + 8192)) == 3
    f32 = _desc(heads=8, head_dim=64, q_dtype=hs.HS2_F32, kv_dtype=hs.HS2_F32, n_q=64, max_ctx=64)
    assert hs.hs2_full_attn_launches(f32) == 2
    assert hs.hs2_full_attn_launches(_desc(head_dim=96)) == 0


def test_long_decode_workspace_holds_the_selection_state(L):
    # rows of 393217 keys and more select from per-sequence histograms and lists in the
    # workspace: 3072 counts, 4 counters, `budget` positions and 4096 8-byte keys per sequence
    short = hs.hs2_workspace_size(_desc(batch=2, max_ctx=393216), False)
    long_ = hs.hs2_workspace_size(_desc(batch=2, max_ctx=393217), False)
    per_seq = 3072 * 4 + 4 * 4 + 1024 * 4 + 4096 * 8
    assert long_ - short >= 2 * per_seq
    assert long_ - short < 2 * per_seq + 8192


def test_null_and_misaligned_arguments_are_rejected(L):
    d = _desc()
    vp = ctypes.c_void_p
    null = None
    st = L.hs2_full_attn_select(ctypes.byref(d), null, null, null, null, null, null, null, null,
                                null, null, null, null, 0, null)
    assert st == hs.HS2_ERR_INVALID_ARG
    fake = vp(0x1000)
    odd = vp(0x1008)
    st = L.hs2_full_attn_select(ctypes.byref(d), odd, fake, fake, null, null, fake, fake, null,
                                fake, fake, null, fake, 1 << 30, null)
    assert st == hs.HS2_ERR_INVALID_ARG
    st = L.hs2_full_attn_select(ctypes.byref(d), fake, fake, fake, null, null, fake, fake, null,
                                fake, fake, null, fake, 16, null)
    assert st == hs.HS2_ERR_WORKSPACE
    e4 = _desc(kv_dtype=hs.HS2_E4M3)
    st = L.hs2_sparse_attn(ctypes.byref(e4), fake, fake, fake, null, null, fake, fake, fake, null,
                           fake, 1 << 30, null)
    assert st == hs.HS2_ERR_INVALID_ARG                               # e4m3 needs scales
    st = L.hs2_topk_select(ctypes.byref(d), fake, 10, fake, 1, fake, fake, fake, 1 << 20, null)
    assert st == hs.HS2_ERR_INVALID_ARG                               # row stride < max_ctx
    st = L.hs2_topk_select(ctypes.byref(d), fake, 4096, fake, 0, fake, fake, fake, 1 << 20, null)
    assert st == hs.HS2_ERR_INVALID_ARG                               # block size 0
    st = L.hs2_kv_quantize_fp8(fake, 10, 96, fake, fake, null)
    assert st == hs.HS2_ERR_UNSUPPORTED
    st = L.hs2_kv_quantize_fp8(null, 10, 128, fake, fake, null)
    assert st == hs.HS2_ERR_INVALID_ARG
    bad = _desc(q_dtype=hs.HS2_F32, kv_dtype=hs.HS2_BF16)
    st = L.hs2_sparse_attn(ctypes.byref(bad), fake, fake, fake, null, null, fake, fake, fake, null,
                           fake, 1 << 30, null)
    assert st == hs.HS2_ERR_UNSUPPORTED


def _tool(*cmd):
    import subprocess
    return subprocess.run(list(cmd), capture_output=True, text=True, check=True).stdout


def test_library_has_no_oracle_dependency(L):
    # the product library neither defines nor imports an oracle symbol and does not
    # depend on the oracle's shared object: checked on the dynamic symbol table and the
    # DT_NEEDED entries (the file's bytes also hold device code and are not scanned)
    syms = _tool("nm", "-D", hs.LIB_PATH)
    assert "hs2_full_attn_select" in syms
    assert not re.search(r"\boracle_\w*", syms), "oracle symbol in libhs2.so"
    needed = _tool("readelf", "-d", hs.LIB_PATH)
    assert "NEEDED" in needed
    assert "oracle" not in needed.lower(), "libhs2.so depends on the oracle"
