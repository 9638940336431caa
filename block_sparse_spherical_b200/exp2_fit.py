"""Coefficients of the polynomial exp2 used on the FMA pipe by the fine-attention kernel.

2^x is evaluated as 2^n * p(f) with n = round(x) and f = x - n in [-1/2, 1/2]
(Cody-Waite range reduction: the split is exact in fp32), and p a polynomial
of degree `deg` that minimises the largest relative error |p(f)/2^f - 1| over
[-1/2, 1/2]: the minimax approximation, found with the Remez exchange
algorithm (alternation at deg+2 points). The kernel rounds the result to
bf16 (relative step 2^-8) for the P·V product, so a relative error near
2^-13 (degree 3) is eight times finer than that rounding.

    python -m block_sparse_spherical_b200.exp2_fit [deg]   # prints coefficients and the error
"""
from __future__ import annotations

import sys

import numpy as np


def remez_exp2(deg: int, iters: int = 40):
    """Minimax relative-error polynomial for 2^f on [-1/2, 1/2]; returns (coeffs low..high, max rel error)."""
    a, b = -0.5, 0.5
    k = np.arange(deg + 2)
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * (deg + 1 - k) / (deg + 1))   # Chebyshev extrema
    grid = np.linspace(a, b, 200001)
    c = None
    for _ in range(iters):
        f = np.exp2(x)
        # p(x_i) - f(x_i) = (-1)^i E f(x_i)   (relative error equioscillates)
        A = np.hstack([x[:, None] ** np.arange(deg + 1)[None, :], -((-1.0) ** k * f)[:, None]])
        sol = np.linalg.solve(A, f)
        c = sol[:-1]
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        # new reference: the extrema of the error between its sign changes
        sign = np.sign(err)
        idx = np.concatenate([[0], np.nonzero(np.diff(sign))[0] + 1, [len(grid)]])
        ext = [s + np.argmax(np.abs(err[s:e])) for s, e in zip(idx[:-1], idx[1:])]
        if len(ext) != deg + 2:
            break
        x = grid[np.array(ext)]
    err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    d = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    coeffs, e = remez_exp2(d)
    f32 = coeffs.astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 200001)
    e32 = float(np.max(np.abs(np.polyval(f32.astype(np.float64)[::-1], grid) / np.exp2(grid) - 1.0)))
    print(f"degree {d}: max relative error {e:.3e} (2^{np.log2(e):.2f}); with fp32 coefficients {e32:.3e}")
    for i, v in enumerate(f32):
        print(f"  c{i} = {float(v)!r}  ({float(v).hex()})")
