"""Fit the polynomial the forward kernel uses to evaluate 2^f on the FMA pipe.

Method: Cody and Waite's range reduction ("Software Manual for the Elementary
Functions", 1980): 2^x = 2^j * 2^f with j = round(x) and f = x - j in
[-1/2, 1/2]; 2^j is applied by adding j to the exponent field. 2^f is
approximated by the degree-n polynomial that minimises the maximum RELATIVE
error on [-1/2, 1/2], found with the Remez exchange algorithm (Remez, 1934):
alternate between solving for a polynomial that equioscillates on n+2
reference points and moving the references to the extrema of the error.

Run: python exp2_poly_fit.py [degree]   -- prints the float32 coefficients
(lowest order first) and the maximum relative error after rounding them to
float32, evaluated in float32 Horner form with fused multiply-adds.
"""
from __future__ import annotations

import sys

import numpy as np

LO, HI = -0.5, 0.5


def remez(n: int, iters: int = 50):
    k = np.arange(n + 2)
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k / (n + 1))[::-1]
    grid = np.linspace(LO, HI, 200001)
    coef = None
    for _ in range(iters):
        # p(f_i) - 2^f_i = (-1)^i E 2^f_i  (relative error of equal size, alternating sign)
        A = np.zeros((n + 2, n + 2))
        for i, f in enumerate(ref):
            A[i, : n + 1] = f ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * 2.0 ** f
        sol = np.linalg.solve(A, 2.0 ** ref)
        coef = sol[: n + 1]
        err = (np.polyval(coef[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new references: the extremum of each sign run of the error
        sign = np.sign(err)
        bounds = np.nonzero(np.diff(sign))[0]
        segs = np.split(np.arange(grid.size), bounds + 1)
        ext = [s[np.argmax(np.abs(err[s]))] for s in segs if s.size]
        if len(ext) < n + 2:
            break
        # keep the n+2 largest alternating extrema
        while len(ext) > n + 2:
            drop = 0 if abs(err[ext[0]]) < abs(err[ext[-1]]) else len(ext) - 1
            ext.pop(drop)
        new_ref = grid[ext]
        if np.allclose(new_ref, ref, atol=1e-12):
            break
        ref = new_ref
    return coef


def fma32(a, b, c):
    """float32 fused multiply-add: the exact product and sum, rounded once."""
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def horner32(coef32, f):
    acc = coef32[-1]
    for c in coef32[-2::-1]:
        acc = fma32(acc, f, c)
    return acc


def max_rel_error(coef32, samples=20001):
    fs = np.linspace(LO, HI, samples).astype(np.float32)
    worst = 0.0
    for f in fs:
        v = float(horner32(coef32, f))
        worst = max(worst, abs(v - 2.0 ** float(f)) / 2.0 ** float(f))
    return worst


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = remez(deg)
    c32 = [np.float32(x) for x in c]
    for i, x in enumerate(c32):
        print(f"c{i} = {float(x)!r}f  ({float(x).hex()})")
    print(f"max relative error (float32 Horner, FMA): {max_rel_error(c32):.3e}")
