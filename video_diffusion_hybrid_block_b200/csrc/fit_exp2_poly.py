"""Fits the polynomial the softmax kernel uses to evaluate part of its exp2
terms on the FMA pipe (beside the MUFU ex2 unit).

Method: Cody-Waite style range reduction x = j + f with j = round(x), f in
[-1/2, 1/2], so 2^x = 2^j * 2^f; 2^f is approximated by a degree-3
polynomial whose coefficients minimise the maximum relative error on
[-1/2, 1/2] (Remez exchange on the relative error, started from a
Chebyshev-node least-squares fit). Prints the coefficients as C++ floats.
"""
import numpy as np


def remez_relative(deg=3, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)  # noqa: E731
    k = np.arange(deg + 2)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (deg + 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative equioscillation)
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(xi)
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error in each sign-alternating run
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        cand = grid[idx]
        vals = err[idx]
        # keep deg+2 alternating points with largest magnitude
        pts, sgn = [], []
        for xv, ev in zip(cand, vals):
            s = np.sign(ev)
            if sgn and s == sgn[-1]:
                if abs(ev) > abs(pts[-1][1]):
                    pts[-1] = (xv, ev)
            else:
                pts.append((xv, ev))
                sgn.append(s)
        while len(pts) > deg + 2:
            if abs(pts[0][1]) < abs(pts[-1][1]):
                pts.pop(0)
            else:
                pts.pop()
        if len(pts) == deg + 2:
            x = np.array([p[0] for p in pts])
    return c, np.max(np.abs(err))


if __name__ == "__main__":
    c, e = remez_relative()
    c32 = np.float32(c)
    grid = np.linspace(-0.5, 0.5, 200001)
    p32 = np.polyval(c32[::-1].astype(np.float64), grid)
    print("max relative error (float32 coefficients): %.3e" % np.max(np.abs(p32 / np.exp2(grid) - 1)))
    for i, v in enumerate(c32):
        print(f"constexpr float kExp2C{i} = {float(v)!r}f;")
