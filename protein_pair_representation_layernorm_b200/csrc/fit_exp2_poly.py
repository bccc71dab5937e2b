"""Coefficients of the degree-3 polynomial behind exp2_poly2 (sm100.cuh).

exp2_poly2 evaluates 2^x on the FMA pipe as 2^n * p(f) with n = round(x) and
f = x - n in [-1/2, 1/2].  p is the polynomial of degree 3 with the smallest
maximum RELATIVE error |p(f) - 2^f| / 2^f on [-1/2, 1/2], found here by the
Remez exchange algorithm (equioscillation at 5 points).  Run it to print the
coefficients (c0 .. c3) and the error bound they achieve; sm100.cuh holds them
rounded to fp32.
"""
import numpy as np


def remez_exp2(deg: int = 3, lo: float = -0.5, hi: float = 0.5, iters: int = 50):
    n = deg + 2
    # start from the Chebyshev extrema
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i for the deg+1 coefficients and E
        m = np.zeros((n, n))
        m[:, :deg + 1] = np.vander(x, deg + 1, increasing=True)
        m[:, deg + 1] = -((-1.0) ** np.arange(n)) * np.exp2(x)
        sol = np.linalg.solve(m, np.exp2(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # the new reference: the largest |err| of each run of equal sign
        sign = np.sign(err)
        idx = [0]
        for i in range(1, len(grid)):
            if sign[i] != sign[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) != n:
            break
        x = grid[idx]
    c32 = c.astype(np.float32).astype(np.float64)
    err32 = np.abs(np.polyval(c32[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
    return c, err32.max()


if __name__ == "__main__":
    c, e = remez_exp2()
    print("coefficients c0..c3:", ", ".join(f"{v:.8f}f" for v in c))
    print(f"max relative error on [-1/2, 1/2] with fp32 coefficients: {e:.3e}")
