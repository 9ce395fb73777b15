"""Derive the polynomial the prefill softmax uses for part of its 2^x evaluations.

Method (Cody and Waite's argument reduction, then a minimax polynomial found by
the Remez exchange algorithm):

    x = n + f,  n = round(x) (integer),  f in [-1/2, 1/2]
    2^x = 2^n * 2^f,    2^f ~= p(f) = c0 + c1 f + c2 f^2 + c3 f^3

p minimises the maximum *relative* error |p(f) / 2^f - 1| over [-1/2, 1/2].
The scale 2^n is applied by adding n to the exponent field of p(f).

Run `python exp2_poly.py` to print the coefficients (as float32 hex and
decimal) and the maximum relative error of the float32 Horner evaluation.
The values are written into ex2_poly2 in fa_common.cuh; tests/test_exp2_poly.py
checks that the constants there match this derivation and meet the error bound.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _solve(ref):
    # p(x_i) - 2^{x_i} = (-1)^i E 2^{x_i}  for the DEGREE+2 reference points
    n = DEGREE + 1
    A = np.zeros((n + 1, n + 1))
    b = np.zeros(n + 1)
    for i, x in enumerate(ref):
        A[i, :n] = [x ** k for k in range(n)]
        A[i, n] = -((-1) ** i) * 2.0 ** x
        b[i] = 2.0 ** x
    sol = np.linalg.solve(A, b)
    return sol[:n], sol[n]


def _rel_err(c, x):
    p = np.polyval(c[::-1], x)
    return p / 2.0 ** x - 1.0


def remez(iters=30):
    # start from Chebyshev extrema
    k = np.arange(DEGREE + 2)
    ref = (LO + HI) / 2 + (HI - LO) / 2 * np.cos(np.pi * k / (DEGREE + 1))[::-1]
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        c, _ = _solve(ref)
        e = _rel_err(c, grid)
        # new reference: the extremum of each sign-alternating run
        sign = np.sign(e)
        idx = [0]
        for i in range(1, len(grid)):
            if sign[i] != sign[idx[-1]] and sign[i] != 0:
                idx.append(i)
            elif abs(e[i]) > abs(e[idx[-1]]):
                idx[-1] = i
        if len(idx) < DEGREE + 2:
            break
        # keep the DEGREE+2 consecutive extrema with the largest minimum magnitude
        best = max(range(len(idx) - DEGREE - 1),
                   key=lambda s: min(abs(e[idx[s + t]]) for t in range(DEGREE + 2)))
        ref = grid[idx[best:best + DEGREE + 2]]
    c, _ = _solve(ref)
    return c


def horner_f32(c, f):
    """Evaluate the polynomial in float32 with fused multiply-adds (as the kernel does)."""
    c = [np.float32(v) for v in c]
    f = np.float32(f) if np.isscalar(f) else f.astype(np.float32)
    acc = np.full_like(f, c[DEGREE], dtype=np.float64)
    for k in range(DEGREE - 1, -1, -1):
        acc = (acc * f.astype(np.float64) + np.float64(c[k])).astype(np.float32).astype(np.float64)
    return acc


def exp2_emulated(x, c):
    """Reference model of the kernel's path: n = round(x), f = x - n, p(f) 2^n."""
    x = np.asarray(x, dtype=np.float32)
    n = np.rint(x).astype(np.float32)
    f = (x - n).astype(np.float32)
    return horner_f32(c, f) * 2.0 ** n.astype(np.float64)


def max_rel_error(c):
    x = np.linspace(-30.0, 8.0, 400001).astype(np.float32)
    return float(np.max(np.abs(exp2_emulated(x, c) / 2.0 ** x.astype(np.float64) - 1.0)))


if __name__ == "__main__":
    coef = remez()
    c32 = [np.float32(v) for v in coef]
    for k, v in enumerate(c32):
        print(f"c{k} = {float(v)!r:>24}  ({np.array(v).view(np.uint32):#010x})")
    print(f"max relative error, float32 Horner: {max_rel_error(c32):.3e}")
