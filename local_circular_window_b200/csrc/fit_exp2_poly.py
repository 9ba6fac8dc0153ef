"""Fits the polynomial behind exp2_poly_x2 (clear_fwd.cuh): p(f) ~ 2^f on [-1/2, 1/2], minimising
the maximum RELATIVE error, by the Remez exchange algorithm (equioscillation at n + 2 points).

    python fit_exp2_poly.py        # prints the float32 coefficients and the error of each degree

The forward kernel uses degree 3: c0..c3 = 0.99992806, 0.69326097, 0.24261113, 0.05517167, with a
maximum relative error of 7.5e-5 (2^-13.7), far below the bf16 rounding (2^-9) that P gets next.
Only NumPy is needed.
"""
import numpy as np


def remez(n, a=-0.5, b=0.5, iters=30, grid=200001):
    """Degree-n coefficients (lowest first) and the max relative error of the minimax fit."""
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * np.arange(n + 2)[::-1] / (n + 1))  # Chebyshev start
    xs = np.linspace(a, b, grid)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i at the reference points
        A = np.zeros((n + 2, n + 2))
        for i in range(n + 2):
            A[i, :n + 1] = x[i] ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:n + 1]
        err = (np.polyval(c[::-1], xs) - 2.0 ** xs) / 2.0 ** xs
        # new reference: the alternating extrema of the error curve (endpoints included)
        idx = [0] + [i for i in range(1, grid - 1) if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0] + [grid - 1]
        pts = []
        for xi, ei in zip(xs[idx], err[idx]):
            if pts and np.sign(pts[-1][1]) == np.sign(ei):
                if abs(ei) > abs(pts[-1][1]):
                    pts[-1] = (xi, ei)
            else:
                pts.append((xi, ei))
        while len(pts) > n + 2:
            pts.pop(0 if abs(pts[0][1]) < abs(pts[-1][1]) else -1)
        if len(pts) == n + 2:
            x = np.array([p[0] for p in pts])
    c32 = c.astype(np.float32)
    err32 = (np.polyval(c32.astype(np.float64)[::-1], xs) - 2.0 ** xs) / 2.0 ** xs
    return c32, float(np.abs(err32).max())


if __name__ == "__main__":
    for n in (2, 3, 4):
        c, e = remez(n)
        print(n, [float(v) for v in c], "max rel err %.3e (2^%.1f)" % (e, np.log2(e)))
