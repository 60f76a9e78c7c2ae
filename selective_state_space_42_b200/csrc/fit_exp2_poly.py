"""Fits the polynomial behind exp2_poly() in scan_tma.cu.

p(f) ≈ 2^f on [-1/2, 1/2] with the smallest maximum RELATIVE error, by the
Remez exchange algorithm (Remez 1934; see e.g. Muller, "Elementary Functions",
ch. 3): alternate between solving for the coefficients and an error level E
that make p(f_i)·2^(-f_i) − 1 = (−1)^i·E on n + 2 reference points, and moving
the reference points to the extrema of the resulting error curve, until the
extrema are level. float64 throughout; the coefficients are then rounded to
float32 and the error of the rounded polynomial is reported.

    python fit_exp2_poly.py [degree]      (default 4)
"""
import sys

import numpy as np


def remez_exp2(deg: int, iters: int = 30):
    a, b = -0.5, 0.5
    m = deg + 2
    # start from Chebyshev extrema
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(m)[::-1] / (m - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # p(x_i) − (−1)^i E 2^x_i = 2^x_i  (relative error level E)
        M = np.zeros((m, m))
        for i, xi in enumerate(x):
            M[i, :deg + 1] = xi ** np.arange(deg + 1)
            M[i, deg + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(M, 2.0 ** x)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extrema of err on each sign-alternating segment
        sign_change = np.where(np.diff(np.sign(err)) != 0)[0]
        bounds = np.concatenate(([0], sign_change + 1, [len(grid)]))
        ext = [s + np.argmax(np.abs(err[s:e])) for s, e in zip(bounds[:-1], bounds[1:]) if e > s]
        if len(ext) != m:
            break
        x = grid[ext]
    return c, np.max(np.abs(err))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c, e64 = remez_exp2(deg)
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    p = np.zeros_like(g)
    for ck in c32[::-1]:  # Horner in float32, as the kernel evaluates it
        p = np.float32(p * g + ck)
    e32 = np.max(np.abs(p.astype(np.float64) / 2.0 ** g.astype(np.float64) - 1.0))
    print(f"degree {deg}: max relative error {e64:.3e} (float64 coefficients), "
          f"{e32:.3e} (float32 coefficients, float32 Horner)")
    for k, ck in enumerate(c32):
        print(f"  c{k} = {float(ck)!r}f")
