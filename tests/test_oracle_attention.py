"""Pins for the oracle's attention routines (CPU only).

Each test checks the oracle against something other than itself: PyTorch's
float64 scaled_dot_product_attention and softmax (textbook attention), closed
forms (probability rows sum to one, so head-summed importance sums to H), and
special cases of the method (a budget that covers the whole context turns the
sparse layer into full attention; a zero budget turns it into sliding-window
attention of width W).
"""
import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, mask, scale):
    """torch float64 SDPA with MQA expanded to every head. q [n, H, D], k/v [T, D]."""
    n, H, D = q.shape
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]            # 1, H, n, D
    kt = torch.from_numpy(k)[None, None].expand(1, H, -1, -1)
    vt = torch.from_numpy(v)[None, None].expand(1, H, -1, -1)
    m = torch.from_numpy(mask)[None, None]
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)
    return out[0].permute(1, 0, 2).numpy()


@pytest.mark.parametrize("n_rows,T,H,D,pos0", [(7, 7, 2, 8, 0), (5, 40, 3, 16, 35),
                                               (33, 33, 4, 4, 0), (1, 300, 8, 32, 299)])
def test_full_attn_matches_torch_sdpa(n_rows, T, H, D, pos0):
    q, k, v = _rand((n_rows, H, D), 1), _rand((T, D), 2), _rand((T, D), 3)
    pos = np.arange(pos0, pos0 + n_rows)
    scale = 1.0 / np.sqrt(D)
    o, lse, scores = oracle.full_attn(q, k, v, pos)
    mask = np.arange(T)[None, :] <= pos[:, None]
    ref = _sdpa(q, k, v, mask, scale)
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-12)
    # LSE against torch.logsumexp of the masked logits
    s = torch.einsum("nhd,td->nht", torch.from_numpy(q), torch.from_numpy(k)) * scale
    s = s.masked_fill(~torch.from_numpy(mask)[:, None, :], float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=1e-12, atol=1e-12)
    # importance = head sum of softmax probabilities
    p = torch.softmax(s, dim=-1).sum(dim=1).numpy()
    np.testing.assert_allclose(scores, p, rtol=1e-10, atol=1e-14)


def test_scores_sum_to_heads_and_are_causal():
    n_rows, T, H, D = 20, 50, 5, 8
    q, k, v = _rand((n_rows, H, D), 4), _rand((T, D), 5), _rand((T, D), 6)
    pos = np.arange(30, 50)
    _, _, scores = oracle.full_attn(q * 3.0, k, v, pos)
    np.testing.assert_allclose(scores.sum(axis=1), np.full(n_rows, H), rtol=0, atol=1e-12)
    assert (scores >= 0).all()
    for r, p in enumerate(pos):
        assert (scores[r, p + 1:] == 0).all()


def test_single_head_score_is_probability_vector():
    T, D = 64, 16
    q, k, v = _rand((1, 1, D), 7), _rand((T, D), 8), _rand((T, D), 9)
    _, _, scores = oracle.full_attn(q, k, v, np.array([T - 1]))
    logits = (k @ q[0, 0]) / np.sqrt(D)
    prob = torch.softmax(torch.from_numpy(logits), dim=0).numpy()
    np.testing.assert_allclose(scores[0], prob, rtol=1e-12, atol=1e-15)


def test_large_logits_are_stable():
    # logits of +-700 would overflow exp without the max shift
    T, D = 10, 4
    q = np.zeros((1, 1, D)); q[0, 0, 0] = 700.0 * 2
    k = np.zeros((T, D)); k[3, 0] = 1.0; k[7, 0] = -1.0
    v = _rand((T, D), 10)
    o, lse, scores = oracle.full_attn(q, k, v, np.array([T - 1]))
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    np.testing.assert_allclose(o[0, 0], v[3], atol=1e-12)
    assert scores[0, 3] == pytest.approx(1.0, abs=1e-12)


def test_sparse_with_full_budget_equals_full_attention():
    n_rows, T, H, D, W, K = 12, 60, 3, 8, 8, 64
    q, k, v = _rand((n_rows, H, D), 11), _rand((T, D), 12), _rand((T, D), 13)
    pos = np.arange(T - n_rows, T)
    o_full, lse_full, scores = oracle.full_attn(q, k, v, pos)
    idx, cnt = oracle.select_rows(scores, pos, W, K)
    np.testing.assert_array_equal(cnt, pos + 1)
    o_sp, lse_sp = oracle.sparse_attn(q, k, v, idx, cnt, want_lse=True)
    np.testing.assert_allclose(o_sp, o_full, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse_sp, lse_full, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("W", [1, 4, 16])
def test_sparse_with_zero_budget_is_sliding_window(W):
    n_rows, T, H, D = 25, 25, 2, 8
    q, k, v = _rand((n_rows, H, D), 14), _rand((T, D), 15), _rand((T, D), 16)
    pos = np.arange(T)
    _, _, scores = oracle.full_attn(q, k, v, pos)
    idx, cnt = oracle.select_rows(scores, pos, W, 0)
    o_sp = oracle.sparse_attn(q, k, v, idx, cnt)
    j = np.arange(T)[None, :]
    mask = (j <= pos[:, None]) & (j > pos[:, None] - W)
    ref = _sdpa(q, k, v, mask, 1.0 / np.sqrt(D))
    np.testing.assert_allclose(o_sp, ref, rtol=1e-10, atol=1e-12)


def test_sparse_is_invariant_to_index_order():
    n_rows, T, H, D = 4, 100, 4, 8
    q, k, v = _rand((n_rows, H, D), 17), _rand((T, D), 18), _rand((T, D), 19)
    rng = np.random.default_rng(20)
    idx = np.stack([np.sort(rng.choice(T, 30, replace=False)) for _ in range(n_rows)]).astype(np.int32)
    cnt = np.full(n_rows, 30, dtype=np.int32)
    o1 = oracle.sparse_attn(q, k, v, idx, cnt)
    perm = np.stack([rng.permutation(row) for row in idx]).astype(np.int32)
    o2 = oracle.sparse_attn(q, k, v, perm, cnt)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    # and equals textbook attention restricted to that set
    for r in range(n_rows):
        mask = np.zeros((1, T), dtype=bool); mask[0, idx[r]] = True
        ref = _sdpa(q[r:r + 1], k, v, mask, 1.0 / np.sqrt(D))
        np.testing.assert_allclose(o1[r:r + 1], ref, rtol=1e-10, atol=1e-12)


def test_bridge_matches_numpy_matmul():
    n, dm, D = 37, 96, 16
    x, w = _rand((n, dm), 21), _rand((dm, 2 * D), 22)
    kk, vv = oracle.bridge(x, w, D)
    ref = np.matmul(x, w)
    np.testing.assert_allclose(kk, ref[:, :D], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(vv, ref[:, D:], rtol=1e-12, atol=1e-12)


def test_hybrid_block_window_always_selected_and_needle_found():
    # a key planted along the query direction must be selected (token level)
    T, H, D, W, K = 400, 4, 16, 16, 32
    rng = np.random.default_rng(23)
    q = rng.standard_normal((1, H, D))
    k = rng.standard_normal((T, D)) / np.sqrt(D)
    v = rng.standard_normal((T, D))
    u = q[0].sum(0); u /= np.linalg.norm(u)
    planted = [5, 77, 200]
    for j in planted:
        k[j] = 4.0 * u
    res = oracle.hybrid_block(q, [q], k, v, np.array([T - 1]), W, K)
    sel = set(res["idx"][0, :res["cnt"][0]].tolist())
    assert set(range(T - W, T)) <= sel
    assert set(planted) <= sel
    assert res["cnt"][0] == W + K
