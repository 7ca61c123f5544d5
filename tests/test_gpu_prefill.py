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


@pytest.mark.parametrize("n_q,ctx", [(300, 300), (300, 1000), (8, 129), (77, 2048 + 5)])
def test_prefill_small_all_rows(n_q, ctx):
    # rows below the window and below the budget, a partial row block, ragged key tiles
    wl = synth.Workload("prefill_case", batch=2, n_q=n_q, ctx=ctx, heads=16, head_dim=128,
                        kv_dtype="bf16", n_sparse=2)
    rep = block_parity(wl, seed=n_q + ctx)
    assert rep["differing_rows"] <= max(2, rep["rows"] // 50)


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
