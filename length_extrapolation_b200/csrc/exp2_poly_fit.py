"""Fit the polynomial used by the kernel's software exp2 (FMA-pipe path).

2^x is evaluated as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]
(range reduction in the manner of Cody and Waite).  2^f is replaced by the
degree-3 polynomial p(f) that minimises the maximum RELATIVE error
|p(f) / 2^f - 1| over [-1/2, 1/2], found with the Remez exchange algorithm
(equioscillation at degree + 2 reference points).  The coefficients are
printed as float32 literals for dca_fwd_sm100.cu; the script also reports the
error of the float32-rounded coefficients.

Usage: python length_extrapolation_b200/csrc/exp2_poly_fit.py
"""
import numpy as np


def remez_relative(deg=3, lo=-0.5, hi=0.5, iters=30):
    n = deg + 2
    # start from Chebyshev extrema mapped to [lo, hi]
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * -np.cos(np.pi * np.arange(n) / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i * E * 2^x_i
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extremum of each sign-alternating run of the error
        s = np.sign(err)
        runs = np.split(np.arange(len(grid)), np.nonzero(np.diff(s))[0] + 1)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) < n:
            break
        # keep the n consecutive extrema with the largest minimum magnitude
        best = max(range(len(ext) - n + 1), key=lambda k: min(abs(err[ext[k:k + n]])))
        x = grid[ext[best:best + n]]
    return c, float(np.max(np.abs(err)))


def main():
    c, e = remez_relative()
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 200001)
    e32 = float(np.max(np.abs(np.polyval(c32.astype(np.float64)[::-1], g) / 2.0 ** g - 1.0)))
    print(f"max relative error (exact coefficients) {e:.3e}, (fp32 coefficients) {e32:.3e}")
    for k, v in enumerate(c32):
        print(f"  c{k} = {float(v)!r:>24}  ({v.view(np.uint32):#010x})")


if __name__ == "__main__":
    main()
