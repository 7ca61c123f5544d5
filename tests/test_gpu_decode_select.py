"""Decode selection, bit for bit against the exact top-K of the call's own importance rows.

Rows up to 393216 keys take the cluster select, longer ones the selection from the attention
kernels' histograms; the cases below cover both.

A decode call of hs2_full_attn_select returns the importance rows it computed (fp32) and the
selection it took from them: the K best candidates of [0, p - W] (importance desc, position
asc) plus the window.  The selection is integer work on those values, so it must equal the
oracle's select_rows run on the same fp32 values exactly -- for spread importance, for tied
groups of keys (identical rows give identical importance; the position decides), for one
value everywhere, on the single-launch path (up to 148 x 4096 keys per wave) and on the
two-kernel path (longer contexts), with ragged positions (rows below the window, rows with
no more candidates than K, rows with one more).  The importance itself is checked against
the oracle elsewhere; here the CUDA selection is pinned to the definition of the selection.
"""
import numpy as np
import pytest
import torch

import kv_shared_b200 as hs
import oracle

pytestmark = pytest.mark.gpu


def _run(kdist, B, T, pos0=None, kv=hs.HS2_BF16, W=128, K=1024, seed=0):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    q = torch.randn(B, 1, 16, 128, generator=g, device="cuda").to(torch.bfloat16)
    if kdist == "normal":
        k = torch.randn(B, T, 128, generator=g, device="cuda")
    elif kdist == "flat":                       # tiny logits: importance within a few percent
        k = torch.randn(B, T, 128, generator=g, device="cuda") * 128 ** -0.5
    elif kdist == "groups":                     # every key one of 5 rows: 5 importance values
        base = torch.randn(5, 128, generator=g, device="cuda")
        k = base[torch.randint(0, 5, (B, T), generator=g, device="cuda")]
    else:                                       # "zero": every logit 0, every importance equal
        k = torch.zeros(B, T, 128, device="cuda")
    v = torch.randn(B, T, 128, generator=g, device="cuda")
    ks = vs = None
    if kv == hs.HS2_E4M3:
        kc = torch.empty(B, T, 128, dtype=torch.uint8, device="cuda")
        vc = torch.empty_like(kc)
        ks = torch.empty(B, T, dtype=torch.float32, device="cuda")
        vs = torch.empty_like(ks)
        hs.hs2_kv_quantize_fp8(k.contiguous(), B * T, 128, kc, ks)
        hs.hs2_kv_quantize_fp8(v.contiguous(), B * T, 128, vc, vs)
        k, v = kc, vc
    else:
        k, v = k.to(torch.bfloat16), v.to(torch.bfloat16)
    pos = np.full(B, T - 1) if pos0 is None else np.asarray(pos0)
    desc = hs.make_desc(B, 1, 16, 128, window=W, budget=K, kv_dtype=kv, max_ctx=T)
    ws = hs.alloc_workspace(desc, scores_in_workspace=False)
    o = torch.empty_like(q)
    idx = torch.empty(B, 1, desc.idx_stride, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, 1, dtype=torch.int32, device="cuda")
    scores = torch.zeros(B, 1, T, dtype=torch.float32, device="cuda")
    q_pos0 = torch.tensor(pos, dtype=torch.int32, device="cuda")
    for _ in range(2):                          # a second call reuses the workspace as it was left
        hs.hs2_full_attn_select(desc, q, k, v, ks, vs, q_pos0, o, None, idx, cnt, scores, ws)
        assert hs.hs2_last_status(ws) == hs.HS2_OK
        s = scores[:, 0].cpu().numpy().astype(np.float64)
        g_idx, g_cnt = idx[:, 0].cpu().numpy(), cnt[:, 0].cpu().numpy()
        for b in range(B):
            o_idx, o_cnt = oracle.select_rows(s[b:b + 1], pos[b:b + 1], W, K, cap=desc.idx_stride)
            assert g_cnt[b] == o_cnt[0], (b, g_cnt[b], o_cnt[0])
            np.testing.assert_array_equal(g_idx[b], o_idx[0], err_msg=f"sequence {b}")


def test_spread_many_waves():
    _run("normal", 32, 131072)                  # 8 waves of 4 sequences x 37 splits


def test_flat_rows_refined():
    # keys like the 128K decode workload's on rows long enough for the histogram selection:
    # the K-th best sits in a coarse bin with most of the row, which the row's CTAs refine
    # together by the next bits of the values
    _run("flat", 2, 400000, seed=8)


def test_ragged_positions():
    # no candidates (p < W), exactly K candidates, K + 1, and long rows in one call
    _run("normal", 6, 50000, pos0=[0, 100, 1151, 1152, 20000, 49999], seed=1)


def test_tied_groups_in_shared_memory():
    _run("groups", 2, 16000, seed=2)            # ~3200 keys per value: the cutoff bin fits


def test_tied_groups_past_the_tie_buffer():
    _run("groups", 1, 400000, seed=3)           # ~80000 keys per value: narrowed over the row


@pytest.mark.parametrize("T", [3000, 30000])
def test_one_value_everywhere(T):
    _run("zero", 1, T, seed=4)                  # the lowest positions win


def test_e4m3_single_launch():
    _run("normal", 4, 300000, kv=hs.HS2_E4M3, seed=5)


def test_e4m3_single_launch_long_rows():
    _run("normal", 2, 450000, kv=hs.HS2_E4M3, seed=9)   # one launch, histogram selection


def test_e4m3_two_kernel_path():
    _run("normal", 2, 1 << 20, kv=hs.HS2_E4M3, seed=6)


def test_small_budget_and_window():
    _run("normal", 3, 9000, pos0=[5, 70, 8999], W=16, K=64, seed=7)
