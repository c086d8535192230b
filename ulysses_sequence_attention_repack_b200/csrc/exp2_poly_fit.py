"""Fit the polynomial behind the FMA-pipe exp2 used by the attention softmax.

Method: range reduction x = j + f with j = round(x) (obtained with the
classic "add 1.5 * 2^23" shifter, so f is in [-1/2, 1/2]), then
2^x = 2^j * p(f), where p is the degree-3 polynomial minimising the maximum
RELATIVE error |p(f) / 2^f - 1| on [-1/2, 1/2].  The minimax polynomial is
found with the Remez exchange algorithm (equioscillation at deg + 2 points),
written here from its textbook statement.  The coefficients printed by this
script are the ones in exp2_poly.cuh; run it to reproduce them:

    python exp2_poly_fit.py
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(LO, HI, 200_001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  (relative error equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extrema of the error on each sign-alternating run
        sign = np.sign(err)
        sign[sign == 0] = 1
        idx, start = [], 0
        for i in range(1, grid.size + 1):
            if i == grid.size or sign[i] != sign[start]:
                seg = slice(start, i)
                idx.append(start + int(np.argmax(np.abs(err[seg]))))
                start = i
        if len(idx) < n:
            break
        # keep n alternating extrema with the largest magnitude
        while len(idx) > n:
            if abs(err[idx[0]]) < abs(err[idx[-1]]):
                idx.pop(0)
            else:
                idx.pop()
        x = grid[idx]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez()
    f32 = np.float32(c)
    grid = np.linspace(LO, HI, 100_001)
    e32 = np.max(np.abs(np.polyval(f32.astype(np.float64)[::-1], grid) / 2.0 ** grid - 1.0))
    for i, v in enumerate(f32):
        print(f"c{i} = {float(v):.9e}f  ({float(v).hex()})")
    print(f"max relative error: fp64 coefficients {e:.3e}, fp32 coefficients {e32:.3e}")
