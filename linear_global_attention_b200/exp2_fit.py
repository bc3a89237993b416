"""Coefficients of the FMA-pipe exp2 used for part of the softmax exponentials.

Method (range reduction in the style of Cody and Waite, then a polynomial):
for x <= 8, clamp x to >= -126, split x = j + f with j = round-to-nearest(x)
and f in [-1/2, 1/2]; approximate 2^f by a degree-3 polynomial p(f) and form
2^x = p(f) * 2^j by adding j to the exponent field of p(f). The polynomial
minimises the maximum relative error |p(f) / 2^f - 1| over [-1/2, 1/2]; it is
found by linear programming on a dense grid (variables c0..c3 and the bound e;
constraints |p(f_i) - 2^f_i| <= e * 2^f_i), then the coefficients are rounded
to float32.

    python -m linear_global_attention_b200.exp2_fit      # prints the coefficients

The CUDA kernel carries the printed constants; a CPU test checks that they
equal this fit and bounds the error of the kernel's float32 evaluation.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
GRID = 4001


def fit(degree: int = DEGREE, grid: int = GRID):
    """(float32 coefficients c0..c_degree, LP bound on the max relative error)."""
    from scipy.optimize import linprog
    f = np.linspace(-0.5, 0.5, grid)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)          # [grid, degree + 1]
    # minimise e  s.t.  V c - y <= e y  and  -(V c - y) <= e y
    A = np.vstack([np.hstack([V, -y[:, None]]), np.hstack([-V, -y[:, None]])])
    b = np.concatenate([y, -y])
    cost = np.zeros(degree + 2)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * (degree + 1) + [(0, None)], method="highs")
    assert res.success, res.message
    return res.x[:degree + 1].astype(np.float32), float(res.x[-1])


def fma32(a, b, c):
    """float32 fused multiply-add: the product of two float32 values is exact in
    float64; the sum is rounded once to float64 and then to float32 (the
    double rounding changes the result only on exact float64 ties)."""
    return (np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64)).astype(np.float32)


def exp2_emulated(x, coeffs) -> np.ndarray:
    """The kernel's float32 evaluation, step by step (x: float32 array, values <= 8)."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)                            # 1.5 * 2^23: adding it rounds to an integer
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    c = [np.float32(v) for v in coeffs]
    p = fma32(c[3], f, c[2])
    p = fma32(p, f, c[1])
    p = fma32(p, f, c[0])
    bits = p.view(np.int32) + (t.view(np.int32) << 23)       # j into the exponent field (two's complement)
    return bits.astype(np.int32).view(np.float32)


if __name__ == "__main__":
    c, e = fit()
    for i, v in enumerate(c):
        print(f"c{i} = {float(v)!r}f  ({v.view(np.uint32):#010x})")
    print(f"LP bound on the relative error: {e:.3e}")
