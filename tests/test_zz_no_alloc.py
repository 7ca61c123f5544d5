"""hs2_sparse_attn_noalloc: sparse attention for callers that cannot allocate.

Some callers of this library have no way to allocate device memory where they
call it (a plugin running inside an inference engine that planned all memory up
front, or code that only owns the inputs and outputs it was handed), so they
cannot provide the workspace hs2_sparse_attn needs.  The no-allocation entry
point keeps that scratch in a fixed array inside the library.  These tests call
it through the C ABI and check that, on two calls in a row, its output agrees
with the workspace entry point's on the same inputs within the tolerances of the
other GPU tests, and that a problem too large for the fixed array is refused.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import kv_shared_b200 as hs
from hs2_check import compare_out

pytestmark = pytest.mark.gpu


def _case(batch, n_q, kv, seed, T=4000):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    H, D = 16, 128
    q = torch.randn(batch, n_q, H, D, generator=g, device="cuda").to(torch.bfloat16)
    kf = torch.randn(batch, T, D, generator=g, device="cuda")
    vf = torch.randn(batch, T, D, generator=g, device="cuda")
    desc = hs.make_desc(batch, n_q, H, D, kv_dtype=hs.HS2_BF16 if kv == "bf16" else hs.HS2_E4M3,
                        max_ctx=T)
    ks = vs = None
    if kv == "bf16":
        k, v = kf.to(torch.bfloat16), vf.to(torch.bfloat16)
    else:
        k = torch.empty(batch, T, D, dtype=torch.uint8, device="cuda")
        v = torch.empty_like(k)
        ks = torch.empty(batch, T, device="cuda")
        vs = torch.empty_like(ks)
        hs.hs2_kv_quantize_fp8(kf, batch * T, D, k, ks)
        hs.hs2_kv_quantize_fp8(vf, batch * T, D, v, vs)
    rng = np.random.default_rng(seed)
    idx = np.full((batch, n_q, 1152), -1, dtype=np.int32)
    cnt = np.zeros((batch, n_q), dtype=np.int32)
    for b in range(batch):
        for r in range(n_q):
            c = int(rng.integers(1, 1153))
            idx[b, r, :c] = np.sort(rng.choice(T, c, replace=False))
            cnt[b, r] = c
    return desc, q, k, v, ks, vs, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
# (32, 1), (3, 1): one CTA cluster per row (no split partials); (1, 200): rows split in two,
# partials and counters in the fixed array; (2, 200): one CTA per row
@pytest.mark.parametrize("shape", [(32, 1), (3, 1), (1, 200), (2, 200)])
def test_noalloc_matches_workspace_entry_point_twice(kv, shape):
    batch, n_q = shape
    ws = None
    for call, seed in enumerate((101, 202)):          # two calls in a row, different inputs
        desc, q, k, v, ks, vs, idx, cnt = _case(batch, n_q, kv, seed)
        if ws is None:
            ws = hs.alloc_workspace(desc)
        ref = torch.empty_like(q)
        ref_lse = torch.empty(batch, n_q, 16, device="cuda")
        hs.hs2_sparse_attn(desc, q, k, v, ks, vs, idx, cnt, ref, ref_lse, ws)
        out = torch.full_like(q, float("nan"))
        lse = torch.full((batch, n_q, 16), float("nan"), device="cuda")
        hs.hs2_sparse_attn_noalloc(desc, q, k, v, ks, vs, idx, cnt, out, lse)
        torch.cuda.synchronize()
        assert hs.hs2_last_status(ws) == hs.HS2_OK
        compare_out(out.double().cpu().numpy(), ref.double().cpu().numpy(), kv, f"O call {call}")
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), rtol=1e-5, atol=1e-5)


def test_noalloc_refuses_problems_beyond_its_scratch():
    # 290 decode rows split in two need about 4.8 MB of partials: more than the 4 MiB array
    desc, q, k, v, ks, vs, idx, cnt = _case(290, 1, "bf16", 7, T=1500)
    out = torch.empty_like(q)
    with pytest.raises(hs.HS2Error) as e:
        hs.hs2_sparse_attn_noalloc(desc, q, k, v, ks, vs, idx, cnt, out, None)
    assert e.value.status == hs.HS2_ERR_WORKSPACE
