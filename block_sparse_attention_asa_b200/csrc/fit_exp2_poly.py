"""Fit the degree-3 polynomial p(f) ~ 2^f on f in [-1/2, 1/2] used by the
softmax's FMA-pipe exponential (Cody-Waite reduction 2^x = 2^n * 2^f with
n = round(x), then p(f)).  Minimax in relative error by a Remez exchange on the
error's extrema; prints the coefficients as float32 and the achieved error."""
import numpy as np


def remez(deg=3, a=-0.5, b=0.5, iters=30):
    f = lambda t: np.exp2(t)
    n = deg + 2
    # start from Chebyshev extrema
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E f(x_i) = f(x_i)  (relative error equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        grid = np.linspace(a, b, 200001)
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new extrema: sign changes partition
        idx = [0]
        for k in range(1, len(grid) - 1):
            if (err[k] - err[k - 1]) * (err[k + 1] - err[k]) <= 0:
                idx.append(k)
        idx.append(len(grid) - 1)
        idx = np.array(sorted(set(idx)))
        cand = grid[idx]
        vals = np.abs(err[idx])
        order = np.argsort(-vals)[:n]
        x = np.sort(cand[order])
    return c, np.max(np.abs(err))


if __name__ == "__main__":
    c, e = remez()
    c32 = c.astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    p = np.float32(c32[3])
    for k in (2, 1, 0):
        p = np.float32(p * grid + c32[k])
    rel = np.abs(p.astype(np.float64) / np.exp2(grid.astype(np.float64)) - 1)
    print("coefficients (c0..c3):", [float(v) for v in c32])
    print("max relative error, exact arithmetic: %.3e; float32 Horner: %.3e" % (e, rel.max()))
