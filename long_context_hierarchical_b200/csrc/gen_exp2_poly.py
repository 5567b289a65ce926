"""Coefficients of the polynomial 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on [-1/2, 1/2].

Method: Cody-Waite style range reduction (2^x = 2^n * 2^f with n = round(x),
f = x - n in [-1/2, 1/2]) and a minimax approximation of 2^f in relative
error, found with the Remez exchange algorithm: solve for the coefficients
and the levelled error E on degree+2 alternation points, move the points to
the extrema of the error curve, repeat until the extrema are equal.

The constants in attn_fwd_tc.cu come from `python gen_exp2_poly.py`.
"""
import numpy as np

DEG = 3
A, B = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    # Chebyshev points as the first alternation set
    x = 0.5 * (A + B) + 0.5 * (B - A) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(A, B, 200001)
    for _ in range(iters):
        f = 2.0 ** x
        # p(x_i) - f_i = (-1)^i E f_i   (relative error levelled at E)
        M = np.zeros((n, n))
        for i in range(n):
            M[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            M[i, deg + 1] = -((-1) ** i) * f[i]
        sol = np.linalg.solve(M, f)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new alternation points: extrema of err on each sign run
        idx = []
        start = 0
        sign = np.sign(err)
        for i in range(1, grid.size + 1):
            if i == grid.size or sign[i] != sign[start]:
                seg = slice(start, i)
                idx.append(start + int(np.argmax(np.abs(err[seg]))))
                start = i
        idx = np.array(idx)
        if idx.size > n:  # keep the n largest consecutive alternation
            while idx.size > n:
                if abs(err[idx[0]]) < abs(err[idx[-1]]):
                    idx = idx[1:]
                else:
                    idx = idx[:-1]
        if idx.size == n:
            x = grid[idx]
    return c, np.max(np.abs(err))


if __name__ == "__main__":
    c, e = remez()
    for i, v in enumerate(c):
        print(f"c{i} = {np.float32(v)!r}  ({v:.17g})")
    print(f"max relative error {e:.3e}")
