"""GPU parity of the prefill path (KV-bridge projection on tcgen05, full attention
with importance on tcgen05, selection, sparse layers) against the CPU oracle."""
import numpy as np
import pytest
import torch

import kv_shared_b200 as hs
import oracle
import synth
from hs2_check import block_parity, f64

pytestmark = pytest.mark.gpu


def _bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def _bridge_bound(x, w, ref):
    """Error bound of an fp32-accumulated dot product of length K rounded once to bf16:
    one bf16 ulp of the exact value plus the accumulation bound 2 K 2^-24 sum_m |x_m w_m|
    (absolute, so it covers outputs that cancel to near zero)."""
    K = x.shape[-1]
    return _bf16_ulp(ref) + 2.0 * K * 2.0 ** -24 * (np.abs(x) @ np.abs(w))


@pytest.mark.parametrize("batch,n,d_model,cap", [(2, 300, 256, 1300), (1, 1, 128, 1), (3, 257, 2048, 600)])
def test_bridge_projection(batch, n, d_model, cap):
    g = torch.Generator().manual_seed(n + d_model)
    x = torch.randn(batch, n, d_model, generator=g).to(torch.bfloat16)
    w = (torch.randn(d_model, 256, generator=g) * d_model ** -0.5).to(torch.bfloat16)
    pos0 = torch.tensor([(7 * b + 5) % (cap - n + 1) for b in range(batch)], dtype=torch.int32)
    sentinel = -3.0
    k = torch.full((batch, cap, 128), sentinel, dtype=torch.bfloat16, device="cuda")
    v = torch.full_like(k, sentinel)
    hs.hs2_kv_bridge_proj(x.cuda(), w.cuda(), batch, n, d_model, 128, pos0.cuda(), cap, k, v)
    torch.cuda.synchronize()
    kc, vc = k.double().cpu().numpy(), v.double().cpu().numpy()
    for b in range(batch):
        kk, vv = oracle.bridge(f64(x[b]), f64(w), 128)
        bound = _bridge_bound(f64(x[b]), f64(w), np.concatenate([kk, vv], axis=1))
        p0 = int(pos0[b])
        for got, ref, bd in ((kc[b, p0:p0 + n], kk, bound[:, :128]), (vc[b, p0:p0 + n], vv, bound[:, 128:])):
            assert (np.abs(got - ref) <= bd).all()
            rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
            assert rel < 4e-3
        untouched = np.ones(cap, bool)
        untouched[p0:p0 + n] = False
        assert (kc[b, untouched] == sentinel).all() and (vc[b, untouched] == sentinel).all()


def test_bridge_full_size_sampled():
    wl = synth.PREFILL_AGENT
    inp = synth.make_inputs(synth.shrink(wl, n_sparse=0), seed=1003, device="cuda")
    B, T = wl.batch, wl.ctx
    k = inp.k.clone()
    v = inp.v.clone()
    pos0 = torch.full((B,), T - wl.n_new, dtype=torch.int32, device="cuda")
    hs.hs2_kv_bridge_proj(inp.hidden, inp.w_kv, B, wl.n_new, wl.d_model, 128, pos0, T, k, v)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(0).choice(wl.n_new, 96, replace=False))
    for b in (0, B - 1):
        xs = f64(inp.hidden[b])[rows]
        kk, vv = oracle.bridge(xs, f64(inp.w_kv), 128)
        bound = _bridge_bound(xs, f64(inp.w_kv), np.concatenate([kk, vv], axis=1))
        got_k = k[b, T - wl.n_new + torch.from_numpy(rows).cuda()].double().cpu().numpy()
        got_v = v[b, T - wl.n_new + torch.from_numpy(rows).cuda()].double().cpu().numpy()
        assert (np.abs(got_k - kk) <= bound[:, :128]).all()
        assert (np.abs(got_v - vv) <= bound[:, 128:]).all()


def _e4m3_ordinal(codes):
    """Signed rank of e4m3 codes in value order (sign-magnitude: the low 7 bits rank the
    magnitude); neighbouring values differ by one."""
    c = np.asarray(codes).astype(np.int64)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def _check_bridge_e4m3(x64, w64, got_codes, got_scales, what):
    """GPU e4m3 bridge rows against the oracle's exact rows.

    The GPU quantizes its fp32-accumulated rows, which differ from the exact ones by at
    most E = 2 K 2^-24 sum_m |x_m w_m| per element (the bound the bf16 test uses).  So:
      - scales: within the range the quantizer gives for row maxima amax_exact -+ E;
      - codes: each GPU code lies between the codes of (x_exact -+ E) / s_gpu, with
        s_gpu checked first;
      - and the codes equal the oracle quantizer applied to the exact rows (fp32
        division and rounding, as both sides compute it), except where the exact value
        sits near a rounding midpoint: at most 1% of the elements, each one code away.
    Returns the number of codes that differ from the oracle's."""
    K = x64.shape[1]
    ref_k, ref_v = oracle.bridge(x64, w64, 128)
    A = np.abs(x64) @ np.abs(w64)
    mism = 0
    for part, ref in enumerate((ref_k, ref_v)):
        E = 2.0 * K * 2.0 ** -24 * A[:, part * 128:(part + 1) * 128]
        codes, s_gpu = got_codes[part], got_scales[part].astype(np.float64)
        amax_lo = np.maximum(np.abs(ref) - E, 0).max(axis=1)
        amax_hi = (np.abs(ref) + E).max(axis=1)
        s_lo = (amax_lo.astype(np.float32) / np.float32(448)).astype(np.float64)
        s_hi = (amax_hi.astype(np.float32) / np.float32(448)).astype(np.float64)
        assert ((s_gpu >= s_lo * (1 - 2 ** -23)) & (s_gpu <= s_hi * (1 + 2 ** -23))).all(), what + ": scale"
        lo = oracle.e4m3_encode(np.clip((ref - E) / s_gpu[:, None], -448, 448))
        hi = oracle.e4m3_encode(np.clip((ref + E) / s_gpu[:, None], -448, 448))
        og = _e4m3_ordinal(codes)
        assert ((og >= _e4m3_ordinal(lo)) & (og <= _e4m3_ordinal(hi))).all(), what + ": code outside its interval"
        o_codes, o_scales = oracle.fp8_quantize(ref.astype(np.float32))
        diff = codes != o_codes
        assert (np.abs(og - _e4m3_ordinal(o_codes)) <= 1).all(), what + ": code more than one step away"
        assert diff.mean() <= 0.01, f"{what}: {diff.mean():.4f} of the codes differ from the oracle's"
        assert (np.abs(s_gpu / o_scales - 1) <= 1e-5).all(), what + ": scale differs from the oracle's"
        mism += int(diff.sum())
    return mism


@pytest.mark.parametrize("batch,n,d_model,cap", [(2, 300, 256, 1300), (3, 257, 2048, 600)])
def test_bridge_projection_e4m3(batch, n, d_model, cap):
    g = torch.Generator().manual_seed(n + d_model + 1)
    x = torch.randn(batch, n, d_model, generator=g).to(torch.bfloat16)
    w = (torch.randn(d_model, 256, generator=g) * d_model ** -0.5).to(torch.bfloat16)
    pos0 = torch.tensor([(5 * b + 3) % (cap - n + 1) for b in range(batch)], dtype=torch.int32)
    k = torch.full((batch, cap, 128), 0x5A, dtype=torch.uint8, device="cuda")
    v = torch.full_like(k, 0x5A)
    ks = torch.full((batch, cap), -1.0, device="cuda")
    vs = torch.full_like(ks, -1.0)
    hs.hs2_kv_bridge_proj(x.cuda(), w.cuda(), batch, n, d_model, 128, pos0.cuda(), cap, k, v,
                          kv_dtype=hs.HS2_E4M3, k_scale=ks, v_scale=vs)
    torch.cuda.synchronize()
    kc, vc, ksc, vsc = k.cpu().numpy(), v.cpu().numpy(), ks.cpu().numpy(), vs.cpu().numpy()
    total = 0
    for b in range(batch):
        p0 = int(pos0[b])
        rows = slice(p0, p0 + n)
        total += _check_bridge_e4m3(f64(x[b]), f64(w), (kc[b, rows], vc[b, rows]), (ksc[b, rows], vsc[b, rows]),
                                    f"seq {b}")
        untouched = np.ones(cap, bool)
        untouched[p0:p0 + n] = False
        assert (kc[b, untouched] == 0x5A).all() and (vc[b, untouched] == 0x5A).all()
        assert (ksc[b, untouched] == -1).all() and (vsc[b, untouched] == -1).all()
    print(f"codes differing from the oracle's (near midpoints): {total} of {2 * batch * n * 128}")


def test_bridge_e4m3_full_size_sampled():
    wl = synth.PREFILL_AGENT
    inp = synth.make_inputs(synth.shrink(wl, n_sparse=0), seed=1003, device="cuda")
    B, T = wl.batch, wl.ctx
    k = torch.empty(B, T, 128, dtype=torch.uint8, device="cuda")
    v = torch.empty_like(k)
    ks = torch.empty(B, T, device="cuda")
    vs = torch.empty_like(ks)
    pos0 = torch.full((B,), T - wl.n_new, dtype=torch.int32, device="cuda")
    hs.hs2_kv_bridge_proj(inp.hidden, inp.w_kv, B, wl.n_new, wl.d_model, 128, pos0, T, k, v,
                          kv_dtype=hs.HS2_E4M3, k_scale=ks, v_scale=vs)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(2).choice(wl.n_new, 96, replace=False))
    sel = T - wl.n_new + torch.from_numpy(rows).cuda()
    for b in (0, B - 1):
        _check_bridge_e4m3(f64(inp.hidden[b])[rows], f64(inp.w_kv),
                           (k[b, sel].cpu().numpy(), v[b, sel].cpu().numpy()),
                           (ks[b, sel].cpu().numpy(), vs[b, sel].cpu().numpy()), f"seq {b}")


@pytest.mark.parametrize("n_q,ctx", [(300, 300), (300, 1000), (8, 129), (77, 2048 + 5)])
def test_prefill_small_all_rows(n_q, ctx):
    # rows below the window and below the budget, a partial row block, ragged key tiles
    wl = synth.Workload("prefill_case", batch=2, n_q=n_q, ctx=ctx, heads=16, head_dim=128,
                        kv_dtype="bf16", n_sparse=2)
    rep = block_parity(wl, seed=n_q + ctx)
    assert rep["differing_rows"] <= max(2, rep["rows"] // 50)


@pytest.mark.parametrize("n_q,ctx", [(300, 1000), (8, 129), (77, 2048 + 5)])
def test_prefill_e4m3_small_all_rows(n_q, ctx):
    # FP8 cache ("Xiaomi unveils HySparse2 ...", AINews article: million-token caches in FP8):
    # codes widened exactly to bf16 for the tensor cores, scales applied in fp32
    wl = synth.Workload("prefill_e4m3_case", batch=2, n_q=n_q, ctx=ctx, heads=16, head_dim=128,
                        kv_dtype="e4m3", n_sparse=1)
    rep = block_parity(wl, seed=n_q + ctx + 5)
    assert rep["differing_rows"] <= max(2, rep["rows"] // 50)


def test_prefill_e4m3_agent_full_size_sampled():
    wl = synth.PREFILL_AGENT_FP8
    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([[0, 127, 128, 1151, 1152, 8191], rng.choice(wl.n_q, 14, replace=False)]))
    rep = block_parity(wl, seed=1009, seqs=[0, 3], device="cuda", rows=rows)
    assert rep["differing_rows"] <= max(2, rep["rows"] // 20)


def test_prefill_with_bridge_small():
    wl = synth.shrink(synth.PREFILL_AGENT, batch=2, n_q=200, ctx=1500 + 200, n_new=200, d_model=256,
                      n_sparse=1)
    block_parity(wl, seed=3)


def test_prefill_agent_full_size_sampled():
    wl = synth.PREFILL_AGENT
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([[0, 7, 8, 127, 128, 1151, 1152, 4095, 8191],
                                     rng.choice(wl.n_q, 23, replace=False)]))
    rep = block_parity(wl, seed=1003, seqs=[0, 3], device="cuda", rows=rows)
    assert rep["differing_rows"] <= max(2, rep["rows"] // 20)


def _select_case(q, k, v, n_q, ctx, budget=1024, window=128):
    """Runs the prefill call on one sequence (rows at positions ctx-n_q .. ctx-1) with and
    without the importance rows and checks the selection against the oracle's."""
    from hs2_check import check_selection
    B, H, D = 1, 16, 128
    desc = hs.make_desc(B, n_q, H, D, window, budget, max_ctx=ctx)
    qd = q.to(torch.bfloat16).cuda().contiguous().view(1, n_q, H, D)
    kd = k.to(torch.bfloat16).cuda().contiguous().view(1, ctx, D)
    vd = v.to(torch.bfloat16).cuda().contiguous().view(1, ctx, D)
    q_pos0 = torch.tensor([ctx - n_q], dtype=torch.int32, device="cuda")
    pos = np.arange(ctx - n_q, ctx)
    o_ref, _, sc_ref = oracle.full_attn(f64(qd[0]), f64(kd[0]), f64(vd[0]), pos)
    o_idx, o_cnt = oracle.select_rows(sc_ref, pos, window, budget)
    results = []
    for with_scores in (True, False):
        ws = hs.alloc_workspace(desc, scores_in_workspace=False)
        o = torch.empty_like(qd)
        idx = torch.empty(1, n_q, desc.idx_stride, dtype=torch.int32, device="cuda")
        cnt = torch.empty(1, n_q, dtype=torch.int32, device="cuda")
        scores = torch.zeros(1, n_q, ctx, device="cuda") if with_scores else None
        hs.hs2_full_attn_select(desc, qd, kd, vd, None, None, q_pos0, o, None, idx, cnt, scores, ws)
        assert hs.hs2_last_status(ws) == hs.HS2_OK
        if with_scores:
            from hs2_check import compare_scores
            compare_scores(scores[0].cpu().numpy(), sc_ref, pos)
        g_idx, g_cnt = idx[0].cpu().numpy(), cnt[0].cpu().numpy()
        check_selection(g_idx, g_cnt, o_idx, o_cnt, sc_ref, pos, window)
        results.append(g_idx)
    # the importance rows are an extra output: the selection does not depend on them
    np.testing.assert_array_equal(results[0], results[1])
    return o_idx, results[0]


def test_fused_select_increasing_importance():
    # every key more important than all earlier ones: each key is a candidate when it
    # appears, so the candidate lists hold whole rows
    g = torch.Generator().manual_seed(11)
    n_q, ctx = 48, 5000
    u = torch.randn(128, generator=g)
    u = u / u.norm()
    q = (6.0 * u).expand(n_q, 16, 128).clone()
    c = torch.linspace(0.2, 3.0, ctx)
    k = c[:, None] * u[None, :] + 0.01 * torch.randn(ctx, 128, generator=g)
    v = torch.randn(ctx, 128, generator=g)
    _select_case(q, k, v, n_q, ctx)


def test_fused_select_all_equal_importance():
    # zero keys: every logit 0, every importance equal -> the lowest positions win; the
    # cutoff bin holds all ~5800 candidates, more than the selection sorts in shared memory
    g = torch.Generator().manual_seed(12)
    n_q, ctx = 40, 6000
    q = torch.randn(n_q, 16, 128, generator=g)
    k = torch.zeros(ctx, 128)
    v = torch.randn(ctx, 128, generator=g)
    o_idx, g_idx = _select_case(q, k, v, n_q, ctx)
    np.testing.assert_array_equal(o_idx, g_idx)


@pytest.mark.parametrize("budget", [0, 1, 64, 4096])
def test_fused_select_budgets(budget):
    g = torch.Generator().manual_seed(13 + budget)
    n_q, ctx = 64, 4500
    q = torch.randn(n_q, 16, 128, generator=g)
    k = torch.randn(ctx, 128, generator=g)
    v = torch.randn(ctx, 128, generator=g)
    _select_case(q, k, v, n_q, ctx, budget=budget)


def test_fused_select_long_context_position_lists():
    # rows with more than 262144 candidates: the selection keeps position lists and sorts
    # them instead of using a bitmap of the candidate range
    g = torch.Generator().manual_seed(14)
    n_q, ctx = 6, 270000
    q = torch.randn(n_q, 16, 128, generator=g)
    k = torch.randn(ctx, 128, generator=g)
    v = torch.randn(ctx, 128, generator=g)
    _select_case(q, k, v, n_q, ctx)
