"""Fit p(f) ~ 2^f on [-1/2, 1/2] minimising the maximum RELATIVE error
(Remez exchange on the weighted error), and print fp32 coefficients.

The kernel evaluates 2^x = 2^round(x) * p(x - round(x)) on the FMA pipe for
part of the softmax exponentials; this script is how its coefficients were
obtained. Usage: python gen_exp2_poly.py [degree]
"""
import sys

import numpy as np


def remez_rel(deg, lo=-0.5, hi=0.5, iters=40):
    f = lambda x: np.exp2(x)
    # initial reference: Chebyshev extrema
    k = np.arange(deg + 2)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (deg + 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve sum c_i x^i + (-1)^j E f(x_j) = f(x_j)  (relative error E)
        A = np.zeros((deg + 2, deg + 2))
        for j, xj in enumerate(x):
            A[j, :deg + 1] = xj ** np.arange(deg + 1)
            A[j, deg + 1] = (-1) ** j * f(xj)
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: alternating extrema of err
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = np.array(idx)
        # keep deg+2 points with largest |err| maintaining alternation
        pts = list(idx)
        while len(pts) > deg + 2:
            # merge same-sign neighbours / drop smallest
            signs = np.sign(err[pts])
            merged = False
            for i in range(len(pts) - 1):
                if signs[i] == signs[i + 1]:
                    drop = i if abs(err[pts[i]]) < abs(err[pts[i + 1]]) else i + 1
                    pts.pop(drop)
                    merged = True
                    break
            if not merged:
                if abs(err[pts[0]]) < abs(err[pts[-1]]):
                    pts.pop(0)
                else:
                    pts.pop()
        x = grid[pts]
    return c, np.abs(err).max()


def fp32_eval_error(c, lo=-0.5, hi=0.5):
    c32 = np.array(c, dtype=np.float32)
    xs = np.linspace(lo, hi, 100001).astype(np.float32)
    acc = np.full_like(xs, c32[-1])
    for ci in c32[-2::-1]:
        acc = (acc.astype(np.float64) * xs + ci).astype(np.float32)  # one rounding per FMA
    return np.abs(acc.astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1).max()


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_rel(deg)
    print(f"degree {deg}: max relative error {e:.3e} (real), {fp32_eval_error(c):.3e} (fp32 Horner)")
    for i, ci in enumerate(c):
        print(f"  c{i} = {np.float32(ci)!r}  ({float(np.float32(ci)).hex()})")
