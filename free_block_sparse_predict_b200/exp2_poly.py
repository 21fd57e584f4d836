"""Coefficients of the polynomial 2^f used by the attention softmax.

The softmax evaluates part of its exponentials on the FMA pipe instead of the
MUFU unit.  For x <= 0 the kernel splits x = n + f with n = round(x) (by adding
and subtracting 1.5 * 2^23) and f in [-1/2, 1/2], evaluates p(f) ~ 2^f with a
cubic in Horner form, and multiplies by 2^n by adding n to the exponent field.

This script computes the cubic that minimises the maximum RELATIVE error on
[-1/2, 1/2] (Remez exchange on the weighted error e(f) = (p(f) - 2^f) / 2^f),
rounds the coefficients to float32, and reports the bound.  The kernel embeds
the printed float32 values; run

    python -m free_block_sparse_predict_b200.exp2_poly

to reproduce them.  The relative error (about 7.5e-5, below the fp16 rounding
of P~ at 4.9e-4) is checked against the hardware ex2 on the GPU by the tests.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez(degree: int = DEGREE, iters: int = 30):
    n = degree + 2
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve sum_i c_i x^i - 2^x = (-1)^j E 2^x   at the n reference points
        A = np.zeros((n, n))
        for j, xj in enumerate(x):
            A[j, :degree + 1] = xj ** np.arange(degree + 1)
            A[j, degree + 1] = -((-1) ** j) * 2.0 ** xj
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:degree + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: the extrema of err, one per sign alternation
        sgn = np.sign(err)
        idx = np.flatnonzero(np.diff(sgn) != 0)
        bounds = np.concatenate(([0], idx + 1, [len(grid)]))
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:])
               if b1 > b0]
        if len(ext) >= n:
            # keep the n largest alternating extrema
            ext = sorted(ext, key=lambda i: -abs(err[i]))[:n]
            x = np.sort(grid[ext])
    return c


def float32_coefficients():
    c = remez()
    c32 = c.astype(np.float32)
    grid = np.linspace(LO, HI, 400001)
    p = np.float32(c32[3])
    for ci in c32[2::-1]:
        p = p * grid.astype(np.float32) + ci
    rel = np.abs(p.astype(np.float64) - 2.0 ** grid) / 2.0 ** grid
    return c32, float(rel.max())


if __name__ == "__main__":
    c32, err = float32_coefficients()
    for i, ci in enumerate(c32):
        print(f"c{i} = {float(ci):.9e}f  (0x{np.float32(ci).view(np.uint32):08x})")
    print(f"max relative error on [-0.5, 0.5] in float32 Horner: {err:.3e}")
