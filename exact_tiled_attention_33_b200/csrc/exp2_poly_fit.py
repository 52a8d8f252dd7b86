"""Fit of the degree-3 polynomial that exp2_poly2 (sm100.cuh) uses for 2^f on [-0.5, 0.5].

    python exact_tiled_attention_33_b200/csrc/exp2_poly_fit.py

Minimises the maximum relative error |p(f) / 2^f - 1| over f in [-0.5, 0.5] by the Remez
exchange algorithm (Chebyshev alternation: at the optimum the relative error takes its
maximum magnitude E with alternating signs at n + 2 = 5 points).  Each iteration solves
p(x_i) - 2^(x_i) = (-1)^i E 2^(x_i) for the coefficients and E at the current reference
points, then moves the points to the extrema of the error on a fine grid.  Prints the
coefficients c3, c2, c1, c0 rounded to float32 (the constants in exp2_poly2) and the
maximum relative error before and after that rounding.
"""

from __future__ import annotations

import numpy as np

LO, HI, DEGREE = -0.5, 0.5, 3


def remez(lo=LO, hi=HI, n=DEGREE, grid_points=200001, iterations=30):
    """Coefficients c0..cn (float64) of the minimax-relative-error fit and its error E."""
    # start from the Chebyshev extrema
    xs = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n + 2)[::-1] / (n + 1))
    grid = np.linspace(lo, hi, grid_points)
    c, e = None, None
    for _ in range(iterations):
        a = np.zeros((n + 2, n + 2))
        for i, x in enumerate(xs):
            a[i, :n + 1] = x ** np.arange(n + 1)
            a[i, n + 1] = -((-1.0) ** i) * np.exp2(x)
        sol = np.linalg.solve(a, np.exp2(xs))
        c, e = sol[:n + 1], sol[n + 1]
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        # one extremum per run of equal sign
        runs = np.flatnonzero(np.diff(np.sign(err)) != 0) + 1
        bounds = np.concatenate([[0], runs, [grid.size]])
        ext = [s + int(np.argmax(np.abs(err[s:t]))) for s, t in zip(bounds[:-1], bounds[1:])]
        if len(ext) != n + 2:
            break
        xs = grid[ext]
    return c, abs(e)


def max_rel_error(coeffs_high_first, points=200001):
    f = np.linspace(LO, HI, points)
    p = np.polyval(np.asarray(coeffs_high_first, dtype=np.float64), f)
    return float(np.abs(p / np.exp2(f) - 1.0).max())


def float32_coefficients():
    """c3, c2, c1, c0 rounded to float32, as exp2_poly2 holds them."""
    c, _ = remez()
    return [float(np.float32(v)) for v in c[::-1]]


if __name__ == "__main__":
    c, e = remez()
    c32 = float32_coefficients()
    print("c3, c2, c1, c0 =", ", ".join(repr(v) for v in c32))
    print(f"max relative error: {e:.4g} (float64 coefficients), "
          f"{max_rel_error(c32):.4g} (float32 coefficients)")
