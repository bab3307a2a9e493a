"""Coefficients of the polynomial the attention kernel uses for part of its exp2 work.

2^f on f in [-1/2, 1/2] by a degree-4 polynomial: interpolation at the 5 Chebyshev nodes of the
interval, then a few Remez exchange steps on the relative error (a textbook minimax method).
The kernel evaluates 2^y = 2^n * p(y - n) with n = round(y); p's relative error bound printed
here is far below the fp16 rounding (2^-11) that P gets right after.

Run: python gen_exp2_poly.py
"""
import numpy as np

DEG = 4


def fit():
    # Chebyshev nodes on [-1/2, 1/2]
    k = np.arange(DEG + 1)
    x = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (DEG + 1)))
    c = np.polyfit(x, np.exp2(x), DEG)[::-1]
    # Remez exchange on the relative error e(x) = p(x) / 2^x - 1
    grid = np.linspace(-0.5, 0.5, 200001)
    ref = np.exp2(grid)
    for _ in range(20):
        err = np.polyval(c[::-1], grid) / ref - 1
        # DEG + 2 alternating extrema
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = np.array(idx)
        if len(idx) != DEG + 2:
            break
        xs = grid[idx]
        # solve p(xs_i) - (-1)^i E 2^xs_i = 2^xs_i  for coefficients and E
        A = np.zeros((DEG + 2, DEG + 2))
        for i, xi in enumerate(xs):
            A[i, : DEG + 1] = xi ** np.arange(DEG + 1)
            A[i, DEG + 1] = (-1) ** i * np.exp2(xi)
        sol = np.linalg.solve(A, np.exp2(xs))
        c = sol[: DEG + 1]
    err = np.polyval(c[::-1], grid) / ref - 1
    return c.astype(np.float32), float(np.abs(err).max())


if __name__ == "__main__":
    c, e = fit()
    for i, v in enumerate(c):
        print(f"c{i} = {float(v)!r}f  // {float(v).hex()}")
    print(f"max relative error on [-1/2, 1/2] (float64 evaluation): {e:.3e}")
