"""Fit the polynomial the prefill kernel uses for part of its exponentials.

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]
(Cody and Waite's argument reduction). 2^f is approximated on that interval
by a degree-4 polynomial whose maximum RELATIVE error is minimised with the
Remez exchange algorithm (equioscillation of the weighted error
(p(f) - 2^f) / 2^f). This script runs the exchange in float64 and prints the
coefficients (c0..c4) rounded to float32, together with the error of the
float32 polynomial evaluated in Horner form, the way the kernel evaluates it.

    python -m exact_softmax_attention_causal_b200.csrc.fit_exp2_poly
"""

from __future__ import annotations

import numpy as np

DEGREE = 4
LO, HI = -0.5, 0.5


def remez(degree: int = DEGREE, iters: int = 30):
    n = degree + 2
    # initial reference: Chebyshev extrema mapped to [LO, HI]
    k = np.arange(n)
    xs = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k / (n - 1))[::-1]
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i for the coefficients and E
        A = np.zeros((n, n))
        for i, x in enumerate(xs):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * 2.0 ** x
        coef = np.linalg.solve(A, 2.0 ** xs)[:degree + 1]
        err = (np.polyval(coef[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: the extrema of the error between its sign changes
        sign = np.sign(err)
        idx = np.concatenate([[0], np.nonzero(np.diff(sign))[0] + 1, [len(grid)]])
        ext = [a + int(np.argmax(np.abs(err[a:b]))) for a, b in zip(idx[:-1], idx[1:]) if b > a]
        if len(ext) >= n:
            # keep the n largest alternating extrema
            while len(ext) > n:
                drop = int(np.argmin(np.abs(err[ext])))
                ext.pop(drop)
            xs = grid[ext]
    return coef


def f32_horner_error(coef32, grid):
    c = [np.float32(v) for v in coef32]
    f = grid.astype(np.float32)
    p = np.float32(c[DEGREE])
    for i in range(DEGREE - 1, -1, -1):
        p = (p * f + c[i]).astype(np.float32)
    return np.max(np.abs((p.astype(np.float64) - 2.0 ** grid.astype(np.float64)) / 2.0 ** grid.astype(np.float64)))


def main():
    coef = remez()
    coef32 = coef.astype(np.float32)
    grid = np.linspace(LO, HI, 400001)
    print("coefficients c0..c4 (float32):")
    for i, v in enumerate(coef32):
        print(f"  c{i} = {float(v)!r}  # {np.float32(v).view(np.uint32):#010x}")
    print(f"max relative error, float32 Horner on [{LO}, {HI}]: {f32_horner_error(coef32, grid):.3e}")


if __name__ == "__main__":
    main()
