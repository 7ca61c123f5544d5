"""The streaming selection of the prefill kernels, modelled on the CPU and checked against
brute force.

The second prefill pass keeps, per query row, a list of candidate keys: a key of
[0, p - W] is appended if its importance reaches the row's running bound `thr` when it
appears.  `thr` only rises, and only to the floor of the highest importance bin with at
least K candidates at or above it.  The selection then takes the row's exact top K (value
desc, position asc) from the list alone.  Correct only if every key of the final top K is
in the list and the bin counts are exact from the cutoff bin up; this file replays that
protocol (two warps per row, 128-key tiles split in halves, the bound raised by one warp
every fourth tile from the counts of the candidates appended so far, the kernel's bin
arithmetic on fp32 bit patterns) on random and adversarial rows and compares the result
with a full sort.  It models the kernel's protocol, not its code; the GPU tests run the
kernels themselves.
"""
import numpy as np
from hypothesis import given, settings, strategies as st

SUB = 2                      # mantissa bits in a bin index (4 bins per octave)
NBINS = 32 << SUB
BASE = (127 - 28) << SUB


def imp_bin(v):
    bits = np.asarray(v, dtype=np.float32).view(np.uint32).astype(np.int64)
    return np.clip((bits >> (23 - SUB)) - BASE, 0, NBINS - 1)


def bin_floor(b):
    if b <= 0:
        return np.float32(0.0)
    return np.array([(b + BASE) << (23 - SUB)], dtype=np.uint32).view(np.float32)[0]


def raise_threshold(hist, K, thr):
    cum = 0
    for b in range(NBINS - 1, -1, -1):
        cum += hist[b]
        if cum >= K:
            return max(thr, bin_floor(b)) if b > 0 else thr
    return thr


def stream_candidates(v, last, K, raise_every=4):
    """Pass 2's protocol for one row: returns the list (positions) and the bin counts."""
    n = v.size
    thr = np.float32(0.0) if K > 0 else np.float32(np.inf)
    hist = np.zeros(NBINS, dtype=np.int64)
    cand = []
    n_tiles = (n + 127) // 128
    for i in range(n_tiles):
        # both warps read the bound before either appends (either order of the two warps
        # is possible on the GPU; reading it first is the looser of the two)
        t = thr
        for half in (0, 1):
            for k in range(i * 128 + 64 * half, min(i * 128 + 64 * half + 64, n)):
                if k <= last and v[k] >= t:
                    cand.append(k)
                    hist[imp_bin(v[k])] += 1
        if i % raise_every == raise_every - 1 and i * 128 <= last:
            thr = raise_threshold(hist, K, thr)
    return np.array(cand, dtype=np.int64), hist


def select_from_list(v, cand, hist, kg):
    """cand_select_kernel's decision: the cutoff bin from the counts, higher bins taken
    whole, the cutoff bin resolved by (value desc, position asc)."""
    if kg == 0:
        return np.zeros(0, dtype=np.int64)
    cum, bstar = 0, None
    for b in range(NBINS - 1, -1, -1):
        if cum + hist[b] >= kg:
            bstar = b
            break
        cum += hist[b]
    assert bstar is not None, "fewer candidates than picks"
    need = kg - cum
    bins = imp_bin(v[cand])
    above = cand[bins > bstar]
    assert above.size == cum, "counts above the cutoff bin do not match the list"
    at = cand[bins == bstar]
    assert at.size == hist[bstar]
    order = sorted(at.tolist(), key=lambda k: (-float(v[k]), k))
    return np.sort(np.concatenate([above, np.array(order[:need], dtype=np.int64)]))


def brute_force(v, last, K):
    keys = sorted(range(last + 1), key=lambda k: (-float(v[k]), k))
    return np.sort(np.array(keys[:min(K, last + 1)], dtype=np.int64))


def check(v, W, K):
    v = np.asarray(v, dtype=np.float32)
    p = v.size - 1
    last = p - W
    cand, hist = stream_candidates(v, last, K)
    kg = min(K, max(0, last + 1))
    got = select_from_list(v, cand, hist, kg)
    np.testing.assert_array_equal(got, brute_force(v, last, K) if last >= 0 else np.zeros(0, np.int64))
    return cand.size


def _row(kind, n, rng):
    if kind == "lognormal":
        return rng.lognormal(-8.0, 1.0, n)
    if kind == "narrow":                       # nearly uniform: one or two bins hold all
        return 1e-4 * (1.0 + 1e-3 * rng.standard_normal(n))
    if kind == "increasing":                   # every key the best so far
        return np.linspace(1e-6, 1e-2, n)
    if kind == "decreasing":
        return np.linspace(1e-2, 1e-6, n)
    if kind == "equal":
        return np.full(n, 3.0e-4)
    if kind == "ties":                         # few distinct values
        return rng.choice([1e-5, 2e-5, 2e-5 * (1 + 2 ** -20), 4e-5], n)
    if kind == "spikes":
        x = np.full(n, 1e-7)
        x[rng.choice(n, max(1, n // 50), replace=False)] = rng.uniform(0.1, 1.0, max(1, n // 50))
        return x
    if kind == "zeros":
        x = np.zeros(n)
        x[rng.choice(n, n // 3, replace=False)] = rng.uniform(0, 1e-3, n // 3)
        return x
    raise ValueError(kind)


KINDS = ["lognormal", "narrow", "increasing", "decreasing", "equal", "ties", "spikes", "zeros"]


@settings(max_examples=60, deadline=None)
@given(kind=st.sampled_from(KINDS), n=st.integers(1, 2600), K=st.sampled_from([0, 1, 7, 64, 200]),
       W=st.sampled_from([1, 16, 128]), seed=st.integers(0, 2 ** 31 - 1))
def test_streamed_list_selects_the_exact_top_k(kind, n, K, W, seed):
    check(_row(kind, n, np.random.default_rng(seed)), W, K)


def test_random_rows_keep_few_candidates():
    # the list is a small part of a long random row; the bound tracks the K-th best
    rng = np.random.default_rng(0)
    n, K = 40000, 256
    size = check(rng.lognormal(-10.0, 0.6, n), 128, K)
    assert size < 0.25 * n, size


def test_increasing_row_lists_every_key():
    n = 3000
    v = np.linspace(1e-6, 1e-2, n).astype(np.float32)
    cand, _ = stream_candidates(v, n - 1 - 128, 64)
    assert cand.size == n - 128                  # each key beats all earlier ones


def test_bins_order_like_values_and_floors_are_lower_bounds():
    rng = np.random.default_rng(1)
    v = np.sort(np.concatenate([rng.lognormal(-12, 4, 5000), [0.0, 2.0 ** -40, 15.99, 16.0]])).astype(np.float32)
    b = imp_bin(v)
    assert (np.diff(b) >= 0).all()
    for x, bx in zip(v, b):
        assert bin_floor(int(bx)) <= x
