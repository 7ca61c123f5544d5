"""The prefill kernels' FMA-pipe exponential (exp2_poly2 in csrc/prefill_attn.cu),
emulated bit for bit in float32 on the CPU and checked against float64 2^x.

The kernel takes a share of its exponentials on the FMA pipe: x = j + r with j
the nearest integer (found by adding and subtracting 1.5 * 2^23), 2^r by a
degree-5 polynomial in Horner form with single-rounding FMAs, and 2^j added
into the exponent bits.  Its stated accuracy is a maximum relative error of
2.1e-7 on [-1/2, 1/2]; the range reduction is exact, so the same bound must hold
for every input the kernel feeds it (x in [-125, 0]).  The coefficients are read
from the kernel source, so these tests check the constants the GPU uses, and
they must agree with the committed fit (kv_shared_b200/exp2_poly_fit.py).
"""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.join(ROOT, "kv_shared_b200"))
import exp2_poly_fit as fit  # noqa: E402

BOUND = 2.11e-7                       # the stated 2.1e-7, to the digit it is given


def _kernel_coefficients():
    src = open(os.path.join(ROOT, "kv_shared_b200", "csrc", "prefill_attn.cu")).read()
    body = src[src.index("float2 exp2_poly2("):]
    body = body[:body.index("return make_float2")]
    vals = [float(v) for v in re.findall(r"make_float2\(([-0-9.e]+)f, \1f\)", body)]
    assert len(vals) == 6, vals            # c5 (the seed) first, then c4 .. c0
    return np.array(vals[::-1], dtype=np.float32)   # low to high


def _exp2_poly2(x):
    """float32 emulation of the kernel's routine on a float32 array."""
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)                   # 1.5 * 2^23
    t = (x + magic).astype(np.float32)               # nearest integer, ties to even
    j = (t - magic).astype(np.float32)
    r = (x - j).astype(np.float32)
    p = fit.horner32(_kernel_coefficients(), r)
    bits = p.view(np.uint32).astype(np.int64) + (t.view(np.uint32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_coefficients_are_the_committed_fit():
    k = _kernel_coefficients()
    c = fit.lawson_fit().astype(np.float32)
    # the fit reproduces the kernel's constants to a few float32 ulps
    assert np.all(np.abs(k.astype(np.float64) / c.astype(np.float64) - 1.0) < 1e-6), (k, c)


def test_polynomial_relative_error_on_the_reduced_interval():
    r = np.linspace(-0.5, 0.5, 200001)
    err = fit.max_rel_error(_kernel_coefficients(), r)
    assert err <= BOUND, err
    # and the degree is not oversized: a fit of degree 4 misses the bound by far
    c4 = fit.lawson_fit(degree=4, grid=np.linspace(-0.5, 0.5, 4001), iters=200).astype(np.float32)
    assert fit.max_rel_error(c4, r) > 10 * BOUND


def test_whole_routine_over_the_kernels_input_range():
    x = np.concatenate([np.linspace(-125.0, 0.0, 400001),
                        -np.arange(0, 126, dtype=np.float64) + 0.5,      # halfway points
                        -np.arange(0, 126, dtype=np.float64)]).astype(np.float32)
    got = _exp2_poly2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() <= BOUND, (rel.max(), x[np.argmax(rel)])
    assert np.all(got > 0) and np.all(np.isfinite(got))


def test_clamp_keeps_results_normal():
    x = np.array([-125.0, -126.0, -200.0, -1e30], dtype=np.float32)
    got = _exp2_poly2(x)
    assert np.all(got >= np.float32(2.0 ** -126))
    assert np.all(got <= np.float32(2.0 ** -124))
