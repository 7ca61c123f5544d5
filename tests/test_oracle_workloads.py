"""Oracle on the synthetic workload recipes at small sizes (CPU only).

Statistical expectations that follow from the planted magnitudes: a planted key
along the summed-query direction has a logit far above the noise maximum, so
token-level selection recovers every planted position; the block-level arm can
keep at most floor(1024/64) = 16 blocks, so with one planted token per block it
recovers at most 16 of 64 (selection-granularity comparison of the MiMo-V3 news
flash: groups of 64 were kept whole in the first generation).
"""
import numpy as np
import pytest

import oracle
import synth


def _f64(t):
    return t.double().numpy()


def _run(wl, seed):
    inp = synth.make_inputs(wl, seed=seed)
    b = 0
    q = _f64(inp.q_full[b])
    k, v = _f64(inp.k[b]), _f64(inp.v[b])
    pos = np.arange(wl.q_pos0, wl.ctx)
    o, lse, scores = oracle.full_attn(q, k, v, pos)
    idx, cnt = oracle.select_rows(scores, pos, wl.window, wl.budget, block_size=wl.block_size)
    return inp, idx, cnt, scores


@pytest.mark.parametrize("ctx", [4096, 16384])
def test_token_level_recall_is_complete(ctx):
    wl = synth.shrink(synth.sweep(ctx), heads=16)
    inp, idx, cnt, _ = _run(wl, seed=1005)
    sel = set(idx[0, :cnt[0]].tolist())
    planted = set(inp.needle_pos[0].tolist())
    assert planted <= sel
    assert cnt[0] == 1152


def test_block_level_recall_is_capped():
    wl = synth.sweep(16384, block_size=64)
    inp, idx, cnt, _ = _run(wl, seed=1005)
    sel = set(idx[0, :cnt[0]].tolist())
    planted = inp.needle_pos[0].tolist()
    recall = sum(p in sel for p in planted) / len(planted)
    assert recall <= 16 / 64 + 1e-12
    assert recall >= 15 / 64      # the 16 kept blocks are planted ones
    assert cnt[0] == 1024 + 128


def test_decode_needles_recovered_small():
    wl = synth.shrink(synth.DECODE_128K, batch=1, ctx=8192)
    inp, idx, cnt, scores = _run(wl, seed=1002)
    sel = set(idx[0, :cnt[0]].tolist())
    assert set(inp.needle_pos[0].tolist()) <= sel
    assert abs(scores[0].sum() - 16) < 1e-9
