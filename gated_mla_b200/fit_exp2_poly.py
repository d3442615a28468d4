"""Fit of the cubic that prefill attention uses for half of its softmax
exponentials (``exp2_poly2`` in csrc/ptx.cuh).

    python gated_mla_b200/fit_exp2_poly.py

Method: 2^x = 2^n * 2^f with n = rint(x) and f = x - n in [-1/2, 1/2]. 2^f is
replaced by the cubic c0 + c1 f + c2 f^2 + c3 f^3 that minimises the largest
RELATIVE error max |p(f) / 2^f - 1| on [-1/2, 1/2]: the Remez exchange
algorithm (E. Ya. Remez, 1934) with weight 2^-f. Each pass solves, on five
reference points f_i, the linear system p(f_i) - (-1)^i E 2^{f_i} = 2^{f_i}
for the coefficients and the levelled error E, then moves the reference
points to the extrema of the weighted error found on a dense grid, until the
extrema level out. The coefficients are printed rounded to fp32, as the kernel
holds them, with the relative error of that fp32 polynomial; the multiply by
2^n is exact (an exponent add), so this is also the error of 2^x.
"""
from __future__ import annotations

import numpy as np


def remez_relative(deg: int = 3, lo: float = -0.5, hi: float = 0.5, iters: int = 30):
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (n - 1 - k) / (n - 1))   # Chebyshev extrema
    grid = np.linspace(lo, hi, 200001)
    E = 0.0
    for _ in range(iters):
        f = np.exp2(x)
        A = np.zeros((n, n))
        for j in range(deg + 1):
            A[:, j] = x ** j
        A[:, deg + 1] = -((-1.0) ** k) * f
        sol = np.linalg.solve(A, f)
        c, E = sol[:deg + 1], sol[deg + 1]
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        # new reference: the extreme point of each run of equal sign of the error
        sign = np.sign(err)
        cuts = np.flatnonzero(np.diff(sign) != 0) + 1
        runs = np.split(np.arange(grid.size), cuts)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) != n:   # keep the n largest alternating extrema
            ext = sorted(ext, key=lambda i: -abs(err[i]))[:n]
            ext.sort()
        x = grid[np.array(ext)]
    return c, abs(E)


def fp32_poly_error(c32, n: int = 2_000_001) -> float:
    """Largest relative error of the kernel's Horner evaluation in fp32
    (each step an fp32 fused multiply-add, emulated exactly in fp64 then
    rounded once) over [-1/2, 1/2]."""
    f = np.linspace(-0.5, 0.5, n).astype(np.float32)
    c0, c1, c2, c3 = (np.float32(v) for v in c32)
    fma = lambda a, b, d: (a.astype(np.float64) * b.astype(np.float64) + np.float64(d)).astype(np.float32)
    p = fma(np.full_like(f, c3), f, c2)
    p = fma(p, f, c1)
    p = fma(p, f, c0)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


def main():
    c, E = remez_relative()
    c32 = [float(np.float32(v)) for v in c]
    print("levelled relative error (exact coefficients): %.4g" % E)
    for i, v in enumerate(c32):
        print("c%d = %.17g" % (i, v))
    print("fp32 evaluation, max relative error: %.4g" % fp32_poly_error(c32))


if __name__ == "__main__":
    main()
