#!/usr/bin/env python
"""Fit the polynomial the fused kernel uses to evaluate 2^x on the FMA pipe.

Method (Cody-Waite style range reduction followed by a minimax polynomial):
  x = n + f with n = round(x) (an integer) and f in [-1/2, 1/2];
  2^x = 2^n * 2^f, where 2^n is applied by adding n to the exponent field and
  2^f is approximated by a degree-3 polynomial p(f).
The coefficients minimise the maximum RELATIVE error |p(f) / 2^f - 1| over
[-1/2, 1/2]; they come from the Remez exchange algorithm on that error
function (equioscillation at degree + 2 points), started from Chebyshev
nodes.  Everything is computed here in float64 from the definition of 2^f.

    python gen_exp2_poly.py          # prints the coefficients and the error bound

The printed values are the ones written into fused_fwd.cuh (EXP2_C0..C3);
tests/test_exp2_poly.py re-runs this fit and checks they agree.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _solve(nodes):
    """Coefficients c_0..c_d and level E with p(x_i) - 2^x_i = (-1)^i E 2^x_i."""
    n = DEGREE + 2
    A = np.zeros((n, n))
    b = np.exp2(nodes)
    for i, x in enumerate(nodes):
        A[i, :DEGREE + 1] = x ** np.arange(DEGREE + 1)
        A[i, DEGREE + 1] = -((-1) ** i) * np.exp2(x)
    sol = np.linalg.solve(A, b)
    return sol[:DEGREE + 1], sol[DEGREE + 1]


def rel_err(c, x):
    return np.polyval(c[::-1], x) / np.exp2(x) - 1.0


def remez(iters: int = 30):
    k = np.arange(DEGREE + 2)
    nodes = 0.5 * (LO + HI) - 0.5 * (HI - LO) * np.cos(np.pi * k / (DEGREE + 1))
    grid = np.linspace(LO, HI, 200001)
    c = None
    for _ in range(iters):
        c, _ = _solve(nodes)
        e = rel_err(c, grid)
        # new nodes: one extremum of the error per sign-alternating segment
        sign = np.sign(e)
        idx = np.flatnonzero(np.diff(sign) != 0)
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = [s + np.argmax(np.abs(e[s:t])) for s, t in zip(bounds[:-1], bounds[1:]) if t > s]
        if len(ext) < DEGREE + 2:
            break
        # keep the DEGREE+2 largest consecutive alternating extrema
        ext = np.array(ext)
        while len(ext) > DEGREE + 2:
            drop = 0 if abs(e[ext[0]]) < abs(e[ext[-1]]) else -1
            ext = np.delete(ext, drop)
        new_nodes = grid[ext]
        if np.allclose(new_nodes, nodes, atol=1e-12):
            break
        nodes = new_nodes
    return c, float(np.max(np.abs(rel_err(c, grid))))


if __name__ == "__main__":
    coeffs, err = remez()
    for i, v in enumerate(coeffs):
        print(f"C{i} = {np.float32(v)!r}  ({v!r})")
    print(f"max relative error on [-1/2, 1/2] (float64 evaluation): {err:.3e}")
