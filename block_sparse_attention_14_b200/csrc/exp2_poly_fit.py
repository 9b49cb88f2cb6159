"""Fits the polynomial used by the attention kernel's software exp2.

exp2(x) is split Cody-Waite style into x = n + f with n = round(x) and
f in [-1/2, 1/2]; 2^n goes into the exponent field and 2^f is a polynomial
p(f) of degree 4 whose coefficients minimise the maximum relative error on
[-1/2, 1/2] (Remez exchange algorithm, run here in float64).

    python exp2_poly_fit.py          # prints the coefficients and the error
"""
import numpy as np


def remez_rel(deg: int, a: float = -0.5, b: float = 0.5, iters: int = 30):
    f = lambda x: np.exp2(x)
    # initial reference: Chebyshev extrema
    k = np.arange(deg + 2)
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k[::-1] / (deg + 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E f(x_i) = f(x_i)  (equioscillating relative error)
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(xi)
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error on each sign-alternating segment
        idx = [0]
        sign = np.sign(err)
        seg_starts = np.flatnonzero(np.diff(sign) != 0) + 1
        bounds = np.concatenate([[0], seg_starts, [len(grid)]])
        ext = [lo + np.argmax(np.abs(err[lo:hi])) for lo, hi in zip(bounds[:-1], bounds[1:])]
        if len(ext) >= deg + 2:
            ext = np.array(ext)
            # keep the deg+2 largest alternating extrema
            while len(ext) > deg + 2:
                if abs(err[ext[0]]) < abs(err[ext[-1]]):
                    ext = ext[1:]
                else:
                    ext = ext[:-1]
            x = grid[ext]
    return c, np.abs(err).max()


if __name__ == "__main__":
    c, e = remez_rel(4)
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 100001)
    p32 = np.zeros_like(g, dtype=np.float32)
    for ci in c32[::-1]:
        p32 = p32 * g.astype(np.float32) + ci
    e32 = np.abs(p32.astype(np.float64) / np.exp2(g) - 1).max()
    print("coefficients (c0..c4):", ", ".join(f"{v:.9e}f" for v in c32))
    print(f"max relative error: {e:.3e} (float64 coefficients), {e32:.3e} (float32 Horner)")
