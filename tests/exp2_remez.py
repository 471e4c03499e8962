"""Derivation of the exp2 polynomial used by window_attn.cu (kExp2C0..C3 in sm100.cuh).

Remez exchange for the degree-3 polynomial p minimising max |p(f) - 2^f| / 2^f on [-1/2, 1/2]:
solve p(x_i) - 2^x_i = (-1)^i E 2^x_i on n+2 reference points, move the points to the extrema of
the error, repeat until the error levels.  ``python tests/exp2_remez.py`` prints the coefficients
(float64 and rounded to float32) and the maximum relative error of the fp32 coefficients.
"""
import numpy as np


def remez_exp2(deg: int = 3, a: float = -0.5, b: float = 0.5, iters: int = 30):
    n = deg + 2
    x = np.cos(np.pi * np.arange(n) / (n - 1))[::-1] * (b - a) / 2 + (a + b) / 2
    xs = np.linspace(a, b, 200001)
    c = None
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * np.exp2(x[i])
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], xs) - np.exp2(xs)) / np.exp2(xs)
        cand = [0] + [i for i in range(1, len(xs) - 1)
                      if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0] + [len(xs) - 1]
        groups = []
        for i in cand:
            if groups and np.sign(err[i]) == np.sign(err[groups[-1][0]]):
                groups[-1].append(i)
            else:
                groups.append([i])
        pts = [max(g, key=lambda i: abs(err[i])) for g in groups]
        while len(pts) > n:
            pts = pts[1:] if abs(err[pts[0]]) < abs(err[pts[-1]]) else pts[:-1]
        x = xs[pts]
    return c


def max_rel_err(c, a=-0.5, b=0.5):
    xs = np.linspace(a, b, 200001)
    return float(np.max(np.abs(np.polyval(np.asarray(c, dtype=np.float64)[::-1], xs)
                               - np.exp2(xs)) / np.exp2(xs)))


if __name__ == "__main__":
    c = remez_exp2()
    c32 = np.float32(c)
    print("float64:", [float(v) for v in c])
    print("float32:", [float(v) for v in c32], "max rel err", max_rel_err(c32))
