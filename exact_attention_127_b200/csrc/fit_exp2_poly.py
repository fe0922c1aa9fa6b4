"""Fit the polynomial the kernel uses to compute 2^x on the FMA pipe.

Method (standard, stated here so the constants can be re-derived):
  * Cody-Waite style range reduction: x = n + f with n = round-to-nearest(x)
    (obtained by adding and subtracting 1.5 * 2^23 in fp32), f in [-1/2, 1/2];
    2^x = 2^n * 2^f, and 2^n is applied by adding n to the exponent field.
  * 2^f on [-1/2, 1/2] is approximated by the polynomial of the given degree
    that minimises the maximum RELATIVE error (minimax), found with the Remez
    exchange algorithm in fp64.  The fp64 coefficients are then rounded to
    fp32 and the error of the fp32 Horner evaluation is measured densely.

Run: python fit_exp2_poly.py [degree]   (prints the coefficients and errors)
"""
import sys

import numpy as np


def remez_relative(deg: int, lo: float = -0.5, hi: float = 0.5, iters: int = 60):
    """Minimax polynomial p of degree `deg` for 2^x on [lo, hi], relative error."""
    n = deg + 2                                   # alternation points
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    coef = None
    for _ in range(iters):
        # solve sum_j c_j x_i^j - 2^{x_i} = (-1)^i E 2^{x_i}   (relative error E)
        A = np.zeros((n, n))
        for j in range(deg + 1):
            A[:, j] = x ** j
        A[:, deg + 1] = -((-1.0) ** k) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** x)
        coef = sol[:deg + 1]
        err = np.polyval(coef[::-1], grid) / 2.0 ** grid - 1.0
        # new alternation set: extrema of err between sign changes
        idx = [0]
        for i in range(1, grid.size - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(grid.size - 1)
        idx = np.array(sorted(set(idx)))
        # keep the largest |err| in each run of equal sign, then take n of them
        runs, cur = [], [idx[0]]
        for i in idx[1:]:
            if np.sign(err[i]) == np.sign(err[cur[-1]]):
                cur.append(i)
            else:
                runs.append(cur)
                cur = [i]
        runs.append(cur)
        pts = [max(r, key=lambda i: abs(err[i])) for r in runs]
        while len(pts) > n:   # drop the smaller end point
            if abs(err[pts[0]]) < abs(err[pts[-1]]):
                pts.pop(0)
            else:
                pts.pop()
        if len(pts) < n:
            break
        x = grid[pts]
    return coef


def fp32_eval_error(coef32, lo=-0.5, hi=0.5):
    f = np.linspace(lo, hi, 2000001).astype(np.float32)
    c = [np.float32(v) for v in coef32]
    p = np.float32(c[-1])
    for cj in c[-2::-1]:
        p = (p * f + cj).astype(np.float32)      # Horner with fp32 rounding (fma rounds once;
    ref = np.exp2(f.astype(np.float64))           # this bound is slightly pessimistic)
    return float(np.max(np.abs(p.astype(np.float64) / ref - 1.0)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = remez_relative(deg)
    c32 = np.asarray(c, dtype=np.float32)
    print(f"degree {deg}, coefficients c0..c{deg} (fp32):")
    for i, v in enumerate(c32):
        print(f"  c{i} = {float(v):.9e}f   (hex 0x{np.float32(v).view(np.uint32):08x})")
    grid = np.linspace(-0.5, 0.5, 200001)
    print("max relative error, fp64 coefficients:",
          float(np.max(np.abs(np.polyval(c[::-1], grid) / 2.0 ** grid - 1))))
    print("max relative error, fp32 Horner:", fp32_eval_error(c32))
