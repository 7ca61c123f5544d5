"""hs2_sparse_attn_noalloc: sparse attention for callers that cannot allocate.

Some callers of this library have no way to allocate device memory where they
call it (a plugin running inside an inference engine that planned all memory up
front, or code that only owns the inputs and outputs it was handed), so they
cannot provide the workspace hs2_sparse_attn needs.  The no-allocation entry
point keeps that scratch in a fixed array inside the library.  These tests call
it through the C ABI and check, on two calls in a row and across calls whose
plans differ (so that whatever an earlier call left in the array is met):
  - its output against the CPU oracle, within the tolerances of the other GPU
    tests;
  - bit equality with the workspace entry point where both run the same plan;
  - that row counts whose split partials would not fit the array are served
    (one CTA per row) instead of refused.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import kv_shared_b200 as hs
import oracle
from hs2_check import compare_out

pytestmark = pytest.mark.gpu

H, D = 16, 128


def _case(batch, n_q, kv, seed, T=4000):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    q = torch.randn(batch, n_q, H, D, generator=g, device="cuda").to(torch.bfloat16)
    kf = torch.randn(batch, T, D, generator=g, device="cuda")
    vf = torch.randn(batch, T, D, generator=g, device="cuda")
    desc = hs.make_desc(batch, n_q, H, D, kv_dtype=hs.HS2_BF16 if kv == "bf16" else hs.HS2_E4M3,
                        max_ctx=T)
    ks = vs = None
    if kv == "bf16":
        k, v = kf.to(torch.bfloat16), vf.to(torch.bfloat16)
        kv64 = [(k[b].double().cpu().numpy(), v[b].double().cpu().numpy()) for b in range(batch)]
    else:
        k = torch.empty(batch, T, D, dtype=torch.uint8, device="cuda")
        v = torch.empty_like(k)
        ks = torch.empty(batch, T, device="cuda")
        vs = torch.empty_like(ks)
        hs.hs2_kv_quantize_fp8(kf, batch * T, D, k, ks)
        hs.hs2_kv_quantize_fp8(vf, batch * T, D, v, vs)
        kv64 = []
        for b in range(batch):           # the oracle quantizes the same fp32 source itself
            pair = []
            for src in (kf, vf):
                codes, scales = oracle.fp8_quantize(src[b].cpu().numpy())
                pair.append(oracle.fp8_dequantize(codes, scales))
            kv64.append(tuple(pair))
    rng = np.random.default_rng(seed)
    idx = np.full((batch, n_q, 1152), -1, dtype=np.int32)
    cnt = np.zeros((batch, n_q), dtype=np.int32)
    for b in range(batch):
        for r in range(n_q):
            c = int(rng.integers(1, 1153))
            idx[b, r, :c] = np.sort(rng.choice(T, c, replace=False))
            cnt[b, r] = c
    dev = (desc, q, k, v, ks, vs, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda())
    return dev, (q, kv64, idx, cnt)


def _check_against_oracle(out, lse, host, kv, what):
    q, kv64, idx, cnt = host
    o = out.double().cpu().numpy()
    l_gpu = lse.cpu().numpy()
    for b, (k64, v64) in enumerate(kv64):
        o_ref, lse_ref = oracle.sparse_attn(q[b].double().cpu().numpy(), k64, v64, idx[b], cnt[b],
                                            want_lse=True)
        compare_out(o[b], o_ref, kv, f"{what} seq {b}")
        np.testing.assert_allclose(l_gpu[b], lse_ref, rtol=1e-4, atol=1e-4)


def _noalloc(dev):
    desc, q, k, v, ks, vs, idx, cnt = dev
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:3], float("nan"), device="cuda")
    hs.hs2_sparse_attn_noalloc(desc, q, k, v, ks, vs, idx, cnt, out, lse)
    return out, lse


def _with_workspace(dev):
    desc, q, k, v, ks, vs, idx, cnt = dev
    ws = hs.alloc_workspace(desc)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], device="cuda")
    hs.hs2_sparse_attn(desc, q, k, v, ks, vs, idx, cnt, out, lse, ws)
    torch.cuda.synchronize()
    assert hs.hs2_last_status(ws) == hs.HS2_OK
    return out, lse


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
# (32, 1), (3, 1): one CTA cluster per row (no split partials); (1, 200): rows split in two,
# partials and counters in the fixed array; (2, 200): one CTA per row
@pytest.mark.parametrize("shape", [(32, 1), (3, 1), (1, 200), (2, 200)])
def test_noalloc_matches_oracle_and_workspace_entry_point_twice(kv, shape):
    batch, n_q = shape
    for call, seed in enumerate((101, 202)):          # two calls in a row, different inputs
        dev, host = _case(batch, n_q, kv, seed)
        out, lse = _noalloc(dev)
        torch.cuda.synchronize()
        _check_against_oracle(out, lse, host, kv, f"call {call}")
        # same plan as the workspace entry point: identical bits
        ref, ref_lse = _with_workspace(dev)
        assert torch.equal(out, ref), f"call {call}: output differs from hs2_sparse_attn"
        assert torch.equal(lse, ref_lse), f"call {call}: LSE differs from hs2_sparse_attn"


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
def test_noalloc_across_plans_and_beyond_the_split_scratch(kv):
    # consecutive calls whose plans differ: two-way split (partials and counters in the
    # array), then 256 and 290 decode rows, whose two-way split would need more than the
    # 4 MiB array (served one CTA per row), then one cluster per row, then the split again
    for i, shape in enumerate([(1, 200), (256, 1), (3, 1), (290, 1), (1, 200)]):
        dev, host = _case(*shape, kv, 300 + i, T=1500)
        out, lse = _noalloc(dev)
        torch.cuda.synchronize()
        _check_against_oracle(out, lse, host, kv, f"shape {shape}")
