"""Derives the coefficients of exp2_poly.cuh: the degree-3 polynomial that
minimises the maximum RELATIVE error of p(f) against 2^f on [-1/2, 1/2]
(Remez exchange algorithm), rounded to fp32.

    python exp2_fit.py        # prints the coefficients and the error bound

The kernels compute 2^x as 2^n * p(f) with n = round(x), f = x - n; the
relative error of the result is that of p on [-1/2, 1/2].  This script is
not run by the build; tests/test_exp2_poly.py re-runs it and checks the
constants in the header."""
import numpy as np

DEGREE = 3
A, B = -0.5, 0.5


def remez(deg=DEGREE, a=A, b=B, iters=40, grid=200001):
    n = deg + 2
    k = np.arange(n)
    x = (a + b) / 2 - (b - a) / 2 * np.cos(np.pi * k / (n - 1))  # Chebyshev extrema
    g = np.linspace(a, b, grid)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  (equi-oscillating relative error)
        M = np.zeros((n, n))
        for i in range(n):
            M[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            M[i, deg + 1] = -((-1) ** i) * np.exp2(x[i])
        sol = np.linalg.solve(M, np.exp2(x))
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], g) / np.exp2(g) - 1
        # new reference: the alternating extrema of the error curve
        turn = np.where(np.diff(np.sign(np.diff(err))) != 0)[0] + 1
        cand = np.concatenate(([0], turn, [len(g) - 1]))
        pts = []
        for i in cand:
            if pts and np.sign(err[i]) == np.sign(err[pts[-1]]):
                if abs(err[i]) > abs(err[pts[-1]]):
                    pts[-1] = i
            else:
                pts.append(i)
        while len(pts) > n:
            pts.pop(0 if abs(err[pts[0]]) < abs(err[pts[-1]]) else -1)
        if len(pts) == n:
            x = g[pts]
    return c


def fp32_coefficients():
    return [float(np.float32(v)) for v in remez()]


def max_rel_error(coef, grid=400001):
    """Max relative error of the fp32 Horner evaluation on [-1/2, 1/2]."""
    f = np.linspace(A, B, grid).astype(np.float32)
    c = [np.float32(v) for v in coef]
    p = c[-1]
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + c[k]).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1)))


if __name__ == "__main__":
    c = fp32_coefficients()
    print("coefficients c0..c3:", ", ".join(repr(v) for v in c))
    print("max relative error (fp32 Horner): %.3e" % max_rel_error(c))
