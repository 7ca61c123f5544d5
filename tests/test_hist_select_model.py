"""The histogram selection of long decode rows, modelled on the CPU and checked against brute
force.

The attention kernels count each candidate key of [0, p - W] into a bin of its fp32 bit
pattern (bits >> 21, 4 per octave); the selection then takes every key of the bins above the
cutoff bin b1 (the bin holding the K-th best), and from b1 the `need` best by (value desc,
position asc).  When b1 holds more keys than the tie buffer, the class of a key becomes (bin,
next 11 bits) and the cutoff class is found again from counts of b1's keys; a class still too
large is narrowed over the whole row.  The narrowing takes 8-bit digits of the key
(value bits << 32 | ~position) from the highest bit where the class's keys differ, and keeps
exactly the keys k with (k & mask) >= prefix.  The picks are then sorted by a counting sort into
at most 4096 buckets of positions and ranks within a bucket.  This file replays that protocol
(with a small tie buffer, so that every route is taken on small rows) and compares the result
with a full sort.  It models the kernel's protocol, not its code; the GPU tests run the kernel.
"""
import numpy as np
from hypothesis import given, settings, strategies as st

SHIFT, FINE_BITS = 21, 11
FINE_SHIFT = SHIFT - FINE_BITS
BINS = 1 << (31 - SHIFT)


def dec_bin(bits):
    return np.minimum(bits >> SHIFT, BINS - 1).astype(np.int64)


def value_class(bits, level):
    c = dec_bin(bits)
    return (c << FINE_BITS) | ((bits >> FINE_SHIFT) & ((1 << FINE_BITS) - 1)) if level else c


def cutoff(counts, need):
    """Highest bin whose count with the counts above reaches need: (bin, keys above it)."""
    cum = 0
    for b in range(len(counts) - 1, -1, -1):
        if cum + counts[b] >= need:
            return b, cum
        cum += counts[b]
    return -1, cum


def narrow(keys, need, shift):
    """Digit narrowing of unique 64-bit keys to the `need` largest: returns (mask, prefix)."""
    if need <= 0:
        return (1 << 64) - 1, (1 << 64) - 1
    mask = prefix = 0
    while True:
        live = [k for k in keys if (k & mask) == prefix]
        dh = np.zeros(256, dtype=np.int64)
        for k in live:
            dh[(k >> shift) & 255] += 1
        d, above = cutoff(dh, need)
        if d < 0:
            return mask | (0xFF << shift), prefix
        prefix |= d << shift
        mask |= 0xFF << shift
        cnt, need = dh[d], need - above
        if cnt <= need or shift == 0:
            return mask, prefix
        shift -= 8


def bucket_sort(pos, n_cand, nbuckets=4096):
    sh = 0
    while (n_cand >> sh) >= nbuckets:
        sh += 1
    order = sorted(pos, key=lambda v: v >> sh)          # the scatter into buckets
    out = [0] * len(pos)
    ends = {}
    for i, v in enumerate(order):
        ends[v >> sh] = i + 1
    starts = {}
    for i, v in enumerate(order):
        starts.setdefault(v >> sh, i)
    for v in order:                                       # rank within the bucket
        b = v >> sh
        r = starts[b] + sum(1 for w in order[starts[b]:ends[b]] if w < v)
        out[r] = v
    return out


def hist_select(v, p, W, K, tie_cap):
    v = np.asarray(v, dtype=np.float32)
    n_cand = max(0, p - W + 1)
    kg = min(K, n_cand)
    if kg == 0:
        return []
    if kg == n_cand:
        return list(range(n_cand))
    bits = v[:n_cand].view(np.uint32).astype(np.int64)
    key = lambda i: (int(bits[i]) << 32) | (~i & 0xFFFFFFFF)
    hist = np.bincount(dec_bin(bits), minlength=BINS)     # what the attention kernels count
    b1, above = cutoff(hist, kg)
    assert b1 >= 0
    level, tval, need = 0, b1, kg - above
    if hist[b1] > tie_cap:                                # refinement by the next 11 bits
        in_b1 = dec_bin(bits) == b1
        fine = np.bincount((bits[in_b1] >> FINE_SHIFT) & ((1 << FINE_BITS) - 1), minlength=1 << FINE_BITS)
        f1, above_f = cutoff(fine, need)
        level, tval, need = 1, (b1 << FINE_BITS) | f1, need - above_f
    cls = value_class(bits, level)
    picks = [int(i) for i in np.nonzero(cls > tval)[0]]
    ties = [key(int(i)) for i in np.nonzero(cls == tval)[0]]
    assert len(picks) == kg - need
    if len(ties) <= tie_cap:
        kand = kor = None
        for k in ties:
            kand = k if kand is None else kand & k
            kor = k if kor is None else kor | k
        diff = (kand ^ kor) if ties else 0
        shift = ((diff.bit_length() - 1) & ~7) if diff else 0
    else:                                                 # narrowed over the row
        shift = (32 + (FINE_SHIFT if level else SHIFT) - 1) & ~7
    mask, prefix = narrow(ties, need, shift)
    taken = [k for k in ties if (k & mask) >= prefix]
    assert len(taken) == need, (len(taken), need)
    picks += [(~k) & 0xFFFFFFFF for k in taken]
    return bucket_sort(picks, n_cand)


def brute(v, p, W, K):
    n_cand = max(0, p - W + 1)
    order = sorted(range(n_cand), key=lambda i: (-float(v[i]), i))
    return sorted(order[:min(K, n_cand)])


def _row(kind, n, rng):
    if kind == "spread":
        return rng.lognormal(-12.0, 1.0, n)
    if kind == "flat":                                    # within ~2%: one coarse bin
        return 1e-4 * (1.0 + 0.01 * rng.standard_normal(n))
    if kind == "groups":                                  # a few values, many keys each
        return rng.choice(rng.lognormal(-10.0, 0.5, 5), n)
    if kind == "equal":
        return np.full(n, 3.0e-5)
    if kind == "increasing":
        return np.linspace(1e-7, 1e-3, n)
    if kind == "zeros":
        x = np.zeros(n)
        x[rng.choice(n, n // 3, replace=False)] = rng.uniform(0.0, 1e-3, n // 3)
        return x
    raise ValueError(kind)


KINDS = ["spread", "flat", "groups", "equal", "increasing", "zeros"]


@settings(max_examples=80, deadline=None)
@given(kind=st.sampled_from(KINDS), n=st.integers(1, 3000), K=st.sampled_from([1, 7, 64, 300]),
       W=st.sampled_from([1, 16, 128]), cap=st.sampled_from([4, 64, 4096]), seed=st.integers(0, 2 ** 31 - 1))
def test_histogram_selection_is_the_exact_top_k(kind, n, K, W, cap, seed):
    v = _row(kind, n, np.random.default_rng(seed)).astype(np.float32)
    p = n - 1
    assert hist_select(v, p, W, K, cap) == brute(v, p, W, K)


def test_flat_row_needs_the_refinement():
    # the 128K decode workload's importance: one coarse bin holds nearly all of the row
    v = _row("flat", 20000, np.random.default_rng(1)).astype(np.float32)
    counts = np.bincount(dec_bin(v.view(np.uint32).astype(np.int64)), minlength=BINS)
    assert counts.max() > 0.5 * v.size
    assert hist_select(v, v.size - 1, 128, 1024, 4096) == brute(v, v.size - 1, 128, 1024)


def test_bucket_sort_orders_any_positions():
    rng = np.random.default_rng(2)
    for n_cand in (10, 5000, 1 << 20):
        pos = sorted(set(rng.integers(0, n_cand, 900).tolist()))
        shuffled = list(rng.permutation(pos))
        assert bucket_sort(shuffled, n_cand) == pos
