"""Coefficients of the cubic that approximates 2^f on [-1/2, 1/2] (minimax in relative
error), used by exp2_poly_x2() in sm100.cuh.

Method: Cody-Waite style range reduction x = n + f with n = round(x), 2^x = 2^n * 2^f;
2^f by a degree-3 polynomial whose coefficients come from the Remez exchange algorithm
on the relative error p(f) / 2^f - 1.  Running this script prints the coefficients and
the error bound; the values are pasted into sm100.cuh.

    python exact_io_aware_64_b200/csrc/gen_exp2_poly.py
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # sum_j c_j x_i^j - (-1)^i E 2^{x_i} = 2^{x_i}
        A = np.zeros((n, n))
        for j in range(deg + 1):
            A[:, j] = x ** j
        A[:, deg + 1] = -((-1.0) ** k) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** x)
        c, E = sol[:deg + 1], sol[deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the alternating extrema of the error
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) < 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = np.array(idx)
        if len(idx) >= n:
            # keep the n largest-|err| points with alternating signs (simple selection)
            best = sorted(idx, key=lambda i: -abs(err[i]))[:n]
            x = np.sort(grid[best])
    err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez()
    for j, v in enumerate(c):
        print(f"c{j} = {np.float32(v)!r}")
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
