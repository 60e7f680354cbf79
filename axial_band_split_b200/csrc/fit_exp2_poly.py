"""Fit the polynomial p(f) ~ 2^f on [-1/2, 1/2] used by the attention softmax to evaluate
part of its exponentials on the FMA pipe (Cody-Waite split 2^x = 2^n * 2^f, n = round(x)).

Minimax in relative error, degree 3: p(f) = c0 + c1 f + c2 f^2 + c3 f^3, by Remez exchange
on e(f) = p(f) / 2^f - 1 over [-1/2, 1/2].  Prints the coefficients and the max error.

    python axial_band_split_b200/csrc/fit_exp2_poly.py
"""
import numpy as np


def fit(deg=3, iters=60, lo=-0.5, hi=0.5):
    n = deg + 1                  # unknowns c0..c_deg, plus the levelled error E
    x = 0.5 * (lo + hi) - 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n + 1) / n)
    g = np.linspace(lo, hi, 400001)
    for _ in range(iters):
        # p(x_i) - (-1)^i E 2^x_i = 2^x_i
        A = np.zeros((n + 1, n + 1))
        for i, xi in enumerate(x):
            A[i, :n] = [xi ** k for k in range(n)]
            A[i, n] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:n]
        e = sum(c[k] * g ** k for k in range(n)) / 2.0 ** g - 1
        # new reference: one extremum of e per run of constant sign
        sign = np.sign(e)
        cuts = np.nonzero(np.diff(sign))[0]
        bounds = [0] + list(cuts + 1) + [len(g)]
        ext = [b0 + int(np.argmax(np.abs(e[b0:b1]))) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        while len(ext) > n + 1:              # keep the n + 1 largest, alternating
            k = int(np.argmin([abs(e[j]) for j in ext]))
            ext.pop(k)
        if len(ext) == n + 1:
            x = g[ext]
    return c, float(np.abs(e).max())


if __name__ == "__main__":
    c, err = fit()
    print("coefficients c0..c3:", ", ".join(f"{v:.9f}" for v in c))
    print(f"max relative error: {err:.3e}")
