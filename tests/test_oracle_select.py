"""Pins for the oracle's selection routines (CPU only).

Brute force on tiny inputs (Python's sorted with a (-score, position) key, and
an O(n^2) rank count, both different algorithms from the oracle's qsort), the
invariants the pages fix (the forced window is always in, the count is
min(p + 1, W + K_sel), output ascending and unique), the tie rule, and the
special case block size 1 == token level.
"""
import os

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _brute_tokens(score, p, W, K):
    n_cand = max(p - W + 1, 0)
    g = sorted(range(n_cand), key=lambda j: (-score[j], j))[:K]
    win = list(range(max(p - W + 1, 0), p + 1))
    return sorted(g + win)


def _rank_count_tokens(score, p, W, K):
    # j is a global pick iff fewer than K candidates beat it under (score desc, index asc)
    n_cand = max(p - W + 1, 0)
    picks = []
    for j in range(n_cand):
        better = sum(1 for i in range(n_cand)
                     if score[i] > score[j] or (score[i] == score[j] and i < j))
        if better < K:
            picks.append(j)
    return sorted(picks + list(range(max(p - W + 1, 0), p + 1)))


def _brute_blocks(score, p, W, K, bs):
    n_cand = max(p - W + 1, 0)
    nb = (n_cand + bs - 1) // bs
    bsc = [max(score[j] for j in range(b * bs, min((b + 1) * bs, n_cand))) for b in range(nb)]
    chosen = sorted(range(nb), key=lambda b: (-bsc[b], b))[:K // bs]
    toks = [j for b in chosen for j in range(b * bs, min((b + 1) * bs, n_cand))]
    return sorted(toks + list(range(max(p - W + 1, 0), p + 1)))


@settings(max_examples=300, deadline=None)
@given(p=st.integers(0, 300), W=st.integers(1, 40), K=st.integers(0, 64),
       seed=st.integers(0, 2**31 - 1), coarse=st.booleans())
def test_tokens_match_brute_force(p, W, K, seed, coarse):
    rng = np.random.default_rng(seed)
    score = rng.random(p + 1)
    if coarse:          # many exact ties
        score = np.round(score * 4) / 4
    got = oracle.select_tokens(score, p, W, K).tolist()
    assert got == _brute_tokens(score, p, W, K)
    assert len(got) == min(p + 1, W + K)
    assert got == sorted(set(got))
    assert set(range(max(p - W + 1, 0), p + 1)) <= set(got)


@settings(max_examples=60, deadline=None)
@given(p=st.integers(0, 120), W=st.integers(1, 16), K=st.integers(0, 40),
       seed=st.integers(0, 2**31 - 1))
def test_tokens_match_rank_count(p, W, K, seed):
    score = np.round(np.random.default_rng(seed).random(p + 1) * 8) / 8
    assert oracle.select_tokens(score, p, W, K).tolist() == _rank_count_tokens(score, p, W, K)


@settings(max_examples=200, deadline=None)
@given(p=st.integers(0, 400), W=st.integers(1, 40), bs=st.integers(1, 16),
       K=st.integers(0, 96), seed=st.integers(0, 2**31 - 1))
def test_blocks_match_brute_force(p, W, bs, K, seed):
    score = np.round(np.random.default_rng(seed).random(p + 1) * 16) / 16
    got = oracle.select_blocks(score, p, W, K, bs).tolist()
    assert got == _brute_blocks(score, p, W, K, bs)


@settings(max_examples=100, deadline=None)
@given(p=st.integers(0, 300), W=st.integers(1, 40), K=st.integers(0, 64),
       seed=st.integers(0, 2**31 - 1))
def test_block_size_one_is_token_level(p, W, K, seed):
    score = np.round(np.random.default_rng(seed).random(p + 1) * 4) / 4
    assert (oracle.select_blocks(score, p, W, K, 1).tolist()
            == oracle.select_tokens(score, p, W, K).tolist())


def test_equal_scores_pick_lowest_positions():
    p, W, K = 500, 128, 100
    got = oracle.select_tokens(np.ones(p + 1), p, W, K)
    assert got.tolist() == list(range(K)) + list(range(p - W + 1, p + 1))


def test_dominant_key_is_always_selected():
    rng = np.random.default_rng(3)
    p, W, K = 3000, 128, 1024
    for j in [0, 1, 1500, p - W]:
        score = rng.random(p + 1) * 1e-3
        score[j] = 1.0
        assert j in set(oracle.select_tokens(score, p, W, K).tolist())
        # a key inside the window is not a candidate but is selected anyway
    score = rng.random(p + 1)
    assert p - 5 in set(oracle.select_tokens(score, p, W, K).tolist())


def test_block_max_rule_keeps_whole_block():
    # one important token keeps its whole 64-token block (first-generation rule)
    p, W, K, bs = 64 * 40 + 127, 128, 128, 64
    score = np.zeros(p + 1)
    score[64 * 7 + 13] = 1.0
    score[64 * 30 + 63] = 0.5
    got = set(oracle.select_blocks(score, p, W, K, bs).tolist())
    assert set(range(64 * 7, 64 * 8)) <= got and set(range(64 * 30, 64 * 31)) <= got
    assert len(got) == 2 * 64 + W


def test_golden_selection_counts():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "selection_counts.txt"))
            if l.strip() and not l.startswith("#")]
    rng = np.random.default_rng(5)
    for p_s, cnt_s, ws_s in rows:
        p, cnt, ws = int(p_s), int(cnt_s), int(ws_s)
        score = rng.random(p + 1)
        got = oracle.select_tokens(score, p, 128, 1024)
        assert len(got) == cnt
        assert got[-min(p + 1, 128):].tolist() == list(range(ws, p + 1))


@pytest.mark.parametrize("bs", [64])
def test_select_rows_padding(bs):
    pos = np.array([0, 100, 2000])
    scores = np.random.default_rng(6).random((3, 2001))
    idx, cnt = oracle.select_rows(scores, pos, 128, 1024, block_size=bs)
    assert idx.shape == (3, 1152)
    for r in range(3):
        assert (idx[r, cnt[r]:] == -1).all()
        assert (np.diff(idx[r, :cnt[r]]) > 0).all()
