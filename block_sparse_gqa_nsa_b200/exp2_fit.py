"""Coefficients of the polynomial 2^f that the attention kernels evaluate on the FMA pipe.

The kernels split x = j + f with j = round(x) and f in [-1/2, 1/2], take 2^j from the
exponent field and 2^f from a cubic c0 + c1 f + c2 f^2 + c3 f^3.  The cubic is the
minimax fit of the RELATIVE error p(f) / 2^f - 1 on [-1/2, 1/2], found here by the Remez
exchange algorithm (E. Ya. Remez, 1934): on a reference of deg + 2 points solve the linear
system p(x_i) = 2^x_i (1 + (-1)^i E) for the coefficients and the levelled error E, move
the reference to the extrema of the new error curve, and repeat until it stops moving.

    python -m block_sparse_gqa_nsa_b200.exp2_fit        # prints the float32 coefficients

The literals in csrc/tc_ptx.cuh (poly_exp2_pair) are this script's output rounded to
float32; a CPU test re-runs the fit and compares them bit for bit.
"""
from __future__ import annotations

import numpy as np


def remez_exp2(deg: int = 3, lo: float = -0.5, hi: float = 0.5, grid: int = 200001, iters: int = 40):
    """(coefficients c0..c_deg in float64, levelled relative error |E|, max error on the grid)."""
    n = deg + 2
    ref = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))  # Chebyshev start
    g = np.linspace(lo, hi, grid)
    coef, lev = None, None
    for _ in range(iters):
        a = np.zeros((n, n))
        for i, xi in enumerate(ref):
            a[i, :deg + 1] = xi ** np.arange(deg + 1)
            a[i, deg + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(a, 2.0 ** ref)
        coef, lev = sol[:deg + 1], sol[deg + 1]
        err = np.polyval(coef[::-1], g) / 2.0 ** g - 1.0
        # new reference: the end points and every interior local extremum of the error
        d = np.diff(err)
        turn = np.nonzero(d[:-1] * d[1:] <= 0)[0] + 1
        new = g[np.r_[0, turn, grid - 1]]
        if len(new) != n or np.allclose(new, ref, rtol=0, atol=1e-12):
            if len(new) == n:
                ref = new
            break
        ref = new
    err = np.polyval(coef[::-1], g) / 2.0 ** g - 1.0
    return coef, abs(lev), float(np.abs(err).max())


def float32_coefficients(deg: int = 3):
    coef, _, _ = remez_exp2(deg)
    return [np.float32(c) for c in coef]


if __name__ == "__main__":
    coef, lev, mx = remez_exp2()
    print("levelled relative error %.4g, max on grid %.4g" % (lev, mx))
    for i, c in enumerate(np.float32(coef)):
        print("c%d = %.10gf" % (i, c))
