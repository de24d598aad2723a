"""Fit the polynomial behind the kernels' FMA-pipe exp2.

The attention softmax evaluates part of its exponentials without the MUFU
unit, by Cody-Waite range reduction plus a polynomial (W. J. Cody and
W. Waite, Software Manual for the Elementary Functions, 1980, ch. 6):

    2^x = 2^n * 2^f,   n = round(x),  f = x - n in [-1/2, 1/2]

and 2^f ~ p(f), a degree-``DEG`` polynomial whose maximum *relative* error on
[-1/2, 1/2] is minimised with the Remez exchange algorithm (E. Remez, 1934;
see e.g. J.-M. Muller, Elementary Functions, 3rd ed., ch. 3).  Running this
script prints the
coefficients pasted into ``attn_fwd.cuh`` and their error bound; the test
``tests/test_exp2_poly.py`` re-runs the fit and checks both.
"""
from __future__ import annotations

import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez_rel(deg: int = DEG, iters: int = 40):
    """Minimax p(f) = c0 + c1 f + ... + c_deg f^deg for 2^f, relative error.

    Returns ``(coefficients c0..c_deg, max |p/2^f - 1| on a fine grid)``.
    """
    n = deg + 2                     # unknowns c0..c_deg and the levelled error E
    k = np.arange(n)
    xs = 0.5 * (LO + HI) - 0.5 * (HI - LO) * np.cos(np.pi * k / (n - 1))
    grid = np.linspace(LO, HI, 40001)
    c = None
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i
        A = np.zeros((n, n))
        for i, x in enumerate(xs):
            A[i, :deg + 1] = [x ** j for j in range(deg + 1)]
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** xs)
        c = sol[:deg + 1]
        err = rel_err(c, grid)
        # one extremum of |err| per run of constant sign
        idx = [0]
        for i in range(1, len(grid)):
            if np.sign(err[i]) != np.sign(err[idx[-1]]):
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) < n:
            break
        best = max(range(len(idx) - n + 1), key=lambda s: min(abs(err[j]) for j in idx[s:s + n]))
        new_xs = grid[idx[best:best + n]]
        if np.allclose(new_xs, xs):
            break
        xs = new_xs
    return c, float(np.max(np.abs(rel_err(c, grid))))


def rel_err(c, x):
    p = np.zeros_like(x)
    for cj in reversed(c):
        p = p * x + cj
    return p / 2.0 ** x - 1.0


def horner_f32(coef, f):
    """Evaluate like the kernel: float32 Horner with fused multiply-adds."""
    f = np.asarray(f, dtype=np.float32)
    c = [np.float32(v) for v in coef]
    p = np.full_like(f, c[-1])
    for cj in reversed(c[:-1]):
        p = (p.astype(np.float64) * f + np.float64(cj)).astype(np.float32)
    return p


if __name__ == "__main__":
    coef, e = remez_rel()
    print("max relative error (real arithmetic): %.3e" % e)
    for j, v in enumerate(coef):
        print("c%d = %.9e  (float32 %r)" % (j, v, float(np.float32(v))))
