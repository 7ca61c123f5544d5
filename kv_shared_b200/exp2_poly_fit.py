"""Coefficients of the degree-5 polynomial for 2^r on [-1/2, 1/2] used by the
prefill kernels' FMA-pipe exponential (exp2_poly2 in csrc/prefill_attn.cu).

Method: Lawson's algorithm, i.e. weighted least squares whose weights are
multiplied, every iteration, by the current relative error at each grid point;
the weights concentrate on the error peaks and the fit converges to the
minimax (equioscillating) relative-error polynomial.  The fit runs in float64 on
a dense grid; the coefficients are then rounded to float32 and the float32
Horner form (single-rounding FMA at every step, as fma.rn.f32x2 computes it) is
evaluated on the grid to report its maximum relative error.

Usage: python kv_shared_b200/exp2_poly_fit.py
"""
import numpy as np

DEGREE = 5
GRID = np.linspace(-0.5, 0.5, 20001)


def lawson_fit(degree=DEGREE, grid=GRID, iters=400):
    """Minimax relative-error fit of 2^r by a polynomial (coefficients low to high)."""
    f = np.exp2(grid)
    V = np.vander(grid, degree + 1, increasing=True)
    w = np.full(grid.size, 1.0 / grid.size)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        # relative error: scale rows by 1 / f
        c, *_ = np.linalg.lstsq((V / f[:, None]) * sw[:, None], sw, rcond=None)
        err = np.abs(V @ c / f - 1.0)
        w = w * err
        w /= w.sum()
    return c


def fma32(a, b, c):
    """float32 a * b + c with one rounding: the product of two float32 values is exact in
    float64, and the float64 sum is rounded once more to float32 (the double rounding can
    differ from a single rounding only in rare halfway cases)."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def horner32(coef32, r32):
    """The kernel's Horner chain p = ((((c5 r + c4) r + c3) r + c2) r + c1) r + c0 in float32."""
    p = np.full_like(r32, coef32[-1])
    for c in coef32[-2::-1]:
        p = fma32(p, r32, np.full_like(r32, c))
    return p


def max_rel_error(coef32, grid=GRID):
    r32 = grid.astype(np.float32)
    p = horner32(np.asarray(coef32, dtype=np.float32), r32).astype(np.float64)
    return float(np.max(np.abs(p / np.exp2(r32.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = lawson_fit()
    c32 = c.astype(np.float32)
    for i, x in enumerate(c32):
        print(f"c{i} = {float(x):.8e}")
    print(f"max relative error of the float32 Horner form on [-1/2, 1/2]: {max_rel_error(c32):.3e}")
