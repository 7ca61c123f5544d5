"""GPU parity of the hybrid-block hot path against the CPU oracle, through the C ABI.

Small cases run the oracle on every row (several tiles and a ragged tail);
full-size workloads, in the launch configuration the benchmark times, are checked
on sampled sequences.  Integer work (selection, FP8 codes) is compared exactly
(selection up to ties inside the 1e-6 band); floating point within the stated
tolerances (tests/hs2_check.py).
"""
import numpy as np
import pytest
import torch

import kv_shared_b200 as hs
import oracle
import synth
from hs2_check import (Dev, block_parity as _block_parity, check_selection, compare_out,
                       compare_scores, f64)

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ FP8 quantizer (bit-exact)
@pytest.mark.parametrize("rows,D", [(1000, 128), (37, 64), (1, 128)])
def test_fp8_quantize_bit_exact(rows, D):
    g = torch.Generator().manual_seed(rows)
    x = torch.randn(rows, D, generator=g) * torch.rand(rows, 1, generator=g) * 10
    x[0, :] = 0.0                                   # all-zero row -> scale 1
    if rows > 3:
        x[2, 5] = 1e-30
        x[3, :] = torch.randn(D, generator=g) * 1e-20
    xd = x.cuda()
    codes = torch.empty(rows, D, dtype=torch.uint8, device="cuda")
    scales = torch.empty(rows, dtype=torch.float32, device="cuda")
    hs.hs2_kv_quantize_fp8(xd, rows, D, codes, scales)
    torch.cuda.synchronize()
    oc, osc = oracle.fp8_quantize(x.numpy())
    np.testing.assert_array_equal(codes.cpu().numpy(), oc)
    np.testing.assert_array_equal(scales.cpu().numpy(), osc)


# ------------------------------------------------------------------ selection (bit-exact on fp32 scores)
def _select_case(n_rows, T, pos, W, K, bs, values, seed):
    rng = np.random.default_rng(seed)
    if values == "coarse":
        s = (rng.integers(0, 8, size=(n_rows, T)) / 8.0).astype(np.float32)
    elif values == "signed":
        s = rng.standard_normal((n_rows, T)).astype(np.float32)
    elif values == "increasing":
        s = np.broadcast_to(np.arange(T, dtype=np.float32), (n_rows, T)).copy()
    elif values == "equal":
        s = np.ones((n_rows, T), dtype=np.float32)
    else:
        s = (rng.random((n_rows, T)) * 1e-3).astype(np.float32)
    desc = hs.make_desc(1, n_rows, 16, 128, window=W, budget=K, max_ctx=T,
                        idx_stride=W + K + 3)
    ws = hs.alloc_workspace(desc)
    sd = torch.from_numpy(s).cuda()
    q_pos0 = torch.tensor([pos], dtype=torch.int32, device="cuda")
    idx = torch.empty(n_rows, W + K + 3, dtype=torch.int32, device="cuda")
    cnt = torch.empty(n_rows, dtype=torch.int32, device="cuda")
    hs.hs2_topk_select(desc, sd, T, q_pos0, bs, idx, cnt, ws)
    assert hs.hs2_last_status(ws) == hs.HS2_OK
    o_idx, o_cnt = oracle.select_rows(s.astype(np.float64), np.arange(pos, pos + n_rows), W, K,
                                      block_size=bs, cap=W + K + 3)
    np.testing.assert_array_equal(cnt.cpu().numpy(), o_cnt)
    np.testing.assert_array_equal(idx.cpu().numpy(), o_idx)


@pytest.mark.parametrize("values", ["uniform", "coarse", "signed"])
@pytest.mark.parametrize("bs", [1, 64, 16])
def test_select_bit_exact_small(values, bs):
    # rows at positions 0..299 cover p < W, p == W - 1, few candidates, K >= candidates
    _select_case(300, 300, 0, 32, 64, bs, values, seed=bs)


@pytest.mark.parametrize("values", ["uniform", "coarse"])
def test_select_bit_exact_long_rows(values):
    # 128 + 1024 at contexts that span many rounds of the compaction and a ragged tail
    _select_case(6, 50000, 50000 - 6, 128, 1024, 1, values, seed=7)
    _select_case(3, 70001, 70001 - 3, 128, 1024, 64, values, seed=8)


@pytest.mark.parametrize("values", ["uniform", "coarse", "signed", "increasing", "equal"])
def test_select_bit_exact_streamed_rows(values):
    # enough rows for one CTA per row and more keys than shared memory holds: the keys are
    # streamed from global memory (first digit at the top bits, compaction by warp
    # segments); increasing scores put every pick in the last warp's segment (its buffer
    # overflows: ordered compaction), equal scores crowd one bin (radix over every key)
    _select_case(300, 30001, 30001 - 300, 128, 1024, 1, values, seed=9)


def test_select_all_equal_scores_picks_lowest():
    T, W, K = 5000, 128, 1024
    s = torch.ones(1, T, device="cuda")
    desc = hs.make_desc(1, 1, 16, 128, window=W, budget=K, max_ctx=T)
    ws = hs.alloc_workspace(desc)
    q_pos0 = torch.tensor([T - 1], dtype=torch.int32, device="cuda")
    idx = torch.empty(1, W + K, dtype=torch.int32, device="cuda")
    cnt = torch.empty(1, dtype=torch.int32, device="cuda")
    hs.hs2_topk_select(desc, s, T, q_pos0, 1, idx, cnt, ws)
    want = list(range(K)) + list(range(T - W, T))
    assert idx[0].cpu().tolist() == want and int(cnt[0]) == W + K


# ------------------------------------------------------------------ sparse attention on given indices
@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
@pytest.mark.parametrize("rows_shape", [(4, 1), (1, 200), (2, 300)])   # cluster, 2-way split, one CTA per row
def test_sparse_attn_random_indices(kv, rows_shape):
    B, n_q = rows_shape
    T, H, D = 3000, 16, 128
    wl = synth.Workload("sparse_case", batch=B, n_q=n_q, ctx=T, heads=H, head_dim=D, kv_dtype=kv,
                        n_sparse=1, kv_std=1.0)
    inp = synth.make_inputs(wl, seed=11)
    dev = Dev(inp)
    rng = np.random.default_rng(3)
    stride = 1152
    idx = np.full((B, n_q, stride), -1, dtype=np.int32)
    cnt = np.zeros((B, n_q), dtype=np.int32)
    sizes = [1, 63, 64, 65, 700, 1152, 1000, 129]
    for b in range(B):
        for r in range(n_q):
            c = sizes[(b * n_q + r) % len(sizes)]
            idx[b, r, :c] = np.sort(rng.choice(T, c, replace=False))
            cnt[b, r] = c
    idx_d = torch.from_numpy(idx).cuda()
    cnt_d = torch.from_numpy(cnt).cuda()
    lse = torch.empty(B, n_q, H, device="cuda")
    dev.sparse(0, idx=idx_d, cnt=cnt_d, lse=lse)
    assert dev.status() == hs.HS2_OK
    for b in range(B):
        k, v = dev.kv_f64(b)
        o_ref, lse_ref = oracle.sparse_attn(f64(inp.q_sparse[0][b]), k, v, idx[b], cnt[b], want_lse=True)
        compare_out(f64(dev.o_sparse[0][b]), o_ref, kv)
        np.testing.assert_allclose(lse[b].cpu().numpy(), lse_ref, rtol=1e-4, atol=1e-3)


def test_sparse_attn_bad_index_reports_status():
    T = 1000
    wl = synth.Workload("bad_idx", batch=1, n_q=1, ctx=T, heads=16, head_dim=128, kv_dtype="bf16",
                        n_sparse=1)
    dev = Dev(synth.make_inputs(wl, seed=1))
    idx = torch.full((1, 1, 1152), -1, dtype=torch.int32, device="cuda")
    idx[0, 0, :3] = torch.tensor([5, T + 7, 9], dtype=torch.int32)
    cnt = torch.tensor([[3]], dtype=torch.int32, device="cuda")
    dev.sparse(0, idx=idx, cnt=cnt)
    assert dev.status() == hs.HS2_ERR_INDEX
    assert torch.isfinite(dev.o_sparse[0].float()).all()
    assert dev.status() == hs.HS2_OK          # the word is cleared once read


def test_decode_wait_timeout_reports_status():
    # The splits of a sequence in the single-launch decode wait (bounded, 2 s) on counters in
    # the workspace's status block.  Counters that can never reach their target make every
    # such wait run out: the call must come back with HS2_ERR_TIMEOUT, the context must stay
    # usable, and after hs2_workspace_init the same workspace must give the normal result.
    wl = synth.shrink(synth.DECODE_128K, batch=2, ctx=20000, needles=4)
    dev = Dev(synth.make_inputs(wl, seed=1009))
    dev.full()
    assert dev.status() == hs.HS2_OK
    ref = [t.clone() for t in (dev.o_full, dev.idx, dev.cnt, dev.scores)]
    status_ints = dev.ws[:4096].view(torch.int32)
    status_ints[1:] = -(10 ** 9)                     # every counter far below any split count
    dev.scores.zero_()
    dev.full()
    assert dev.status() == hs.HS2_ERR_TIMEOUT
    hs.hs2_workspace_init(dev.ws)
    dev.full()
    assert dev.status() == hs.HS2_OK
    for got, want in zip((dev.o_full, dev.idx, dev.cnt, dev.scores), ref):
        assert torch.equal(got, want)


# ------------------------------------------------------------------ whole hybrid block
def test_tiny_f32_block_all_rows():
    rep = _block_parity(synth.TINY, seed=1001)
    assert rep["differing_rows"] <= 2


@pytest.mark.parametrize("ctx", [4096 + 77, 1152, 1153, 129, 20000])
def test_decode_bf16_small(ctx):
    wl = synth.shrink(synth.DECODE_128K, batch=3, ctx=ctx, needles=min(16, max(0, ctx - 200) // 10))
    _block_parity(wl, seed=1002)


@pytest.mark.parametrize("batch,ctx", [(40, 20000), (200, 4096 + 77)])
def test_decode_bf16_several_waves(batch, ctx):
    # more sequences than one wave of the single-launch path holds (2 and 3 waves)
    wl = synth.shrink(synth.DECODE_128K, batch=batch, ctx=ctx, needles=16)
    _block_parity(wl, seed=1003)


def test_decode_e4m3_several_waves():
    # e4m3 cache through the single-launch path over three waves (per-wave V scales kept
    # in shared memory, tail tiles of every split)
    wl = synth.shrink(synth.DECODE_1M_FP8, batch=200, ctx=4096 + 77, needles=16)
    _block_parity(wl, seed=1007)


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
def test_decode_ragged_positions(kv):
    # every sequence at its own position: splits past a short sequence's end hold no keys
    base = synth.DECODE_128K if kv == "bf16" else synth.DECODE_1M_FP8
    wl = synth.shrink(base, batch=40, ctx=20000, needles=16)
    rng = np.random.default_rng(7)
    pos0 = rng.integers(0, wl.ctx, size=wl.batch)
    pos0[:8] = [0, 1, 63, 64, 1151, 1152, 2879, wl.ctx - 1]
    _block_parity(wl, seed=1006, pos0=pos0)


def test_decode_fp8_small():
    wl = synth.shrink(synth.DECODE_1M_FP8, batch=2, ctx=16384 + 5)
    _block_parity(wl, seed=1004)


def test_decode_128k_full_size_sampled():
    _block_parity(synth.DECODE_128K, seed=1002, seqs=[0, 31], device="cuda")


def test_decode_1m_fp8_full_size_sampled():
    _block_parity(synth.DECODE_1M_FP8, seed=1004, seqs=[3], device="cuda")


def test_decode_long_rows_ragged():
    # long rows (more splits than one wave's share) with ragged positions: short rows, rows
    # below the window and rows with fewer candidates than the budget in the same call
    wl = synth.shrink(synth.DECODE_128K, batch=6, ctx=400000, needles=16)
    pos0 = np.array([0, 100, 1151, 5000, 393300, wl.ctx - 1])
    _block_parity(wl, seed=1010, pos0=pos0, device="cuda")


def test_decode_long_rows_all_equal_importance():
    # zero keys: every logit 0 and every importance equal, so the lowest positions win; the
    # whole row lands in one bin of the selection histogram, narrowed over the row in memory
    from hs2_check import check_selection
    T = 400000
    g = torch.Generator(device="cuda")
    g.manual_seed(9)
    q = torch.randn(1, 1, 16, 128, generator=g, device="cuda").to(torch.bfloat16)
    k = torch.zeros(1, T, 128, dtype=torch.bfloat16, device="cuda")
    v = torch.randn(1, T, 128, generator=g, device="cuda").to(torch.bfloat16)
    desc = hs.make_desc(1, 1, 16, 128, max_ctx=T)
    ws = hs.alloc_workspace(desc)
    o = torch.empty_like(q)
    idx = torch.empty(1, 1, desc.idx_stride, dtype=torch.int32, device="cuda")
    cnt = torch.empty(1, 1, dtype=torch.int32, device="cuda")
    q_pos0 = torch.tensor([T - 1], dtype=torch.int32, device="cuda")
    hs.hs2_full_attn_select(desc, q, k, v, None, None, q_pos0, o, None, idx, cnt, None, ws)
    assert hs.hs2_last_status(ws) == hs.HS2_OK
    pos = np.array([T - 1])
    _, _, sc = oracle.full_attn(q[0].double().cpu().numpy(), k[0].double().cpu().numpy(),
                                v[0].double().cpu().numpy(), pos)
    o_idx, o_cnt = oracle.select_rows(sc, pos, 128, 1024)
    check_selection(idx[0].cpu().numpy(), cnt[0].cpu().numpy(), o_idx, o_cnt, sc, pos, 128)
    np.testing.assert_array_equal(idx[0].cpu().numpy(), o_idx)


@pytest.mark.parametrize("ctx", [4096, 32768, 262144, 1 << 20])   # 1M: two-kernel decode path
def test_granularity_sweep_recall(ctx):
    tok = synth.sweep(ctx)
    _block_parity(tok, seed=1005, device="cuda")
    blk = synth.sweep(ctx, block_size=64)
    inp = synth.make_inputs(blk, seed=1005, device="cuda")
    dev = Dev(inp)
    dev.full()
    # the block arm runs on the same importance through the block-level selection
    idx = torch.empty_like(dev.idx)
    cnt = torch.empty_like(dev.cnt)
    hs.hs2_topk_select(dev.desc, dev.scores.view(-1, blk.ctx), blk.ctx, dev.q_pos0, 64, idx, cnt, dev.ws)
    assert dev.status() == hs.HS2_OK
    sel = set(idx[0, 0, :int(cnt[0, 0])].cpu().tolist())
    planted = inp.needle_pos[0].tolist()
    recall_blk = sum(p in sel for p in planted) / len(planted)
    assert recall_blk <= 16 / 64 + 1e-9
