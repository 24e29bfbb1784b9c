"""Reproduces the coefficients of the degree-3 polynomial that the attention
kernel's FMA-pipe exponential (exp2_poly_x2 in sm100.cuh) uses for 2^f on
f in [-1/2, 1/2].

Method: Lawson's iteratively reweighted least squares for the minimax
relative error.  On n Chebyshev nodes of [-1/2, 1/2], solve the weighted
least-squares problem min sum_i w_i ((p(f_i) - 2^f_i) / 2^f_i)^2, then
multiply each weight by that node's relative error and renormalise; the
weights concentrate on the equioscillation points and p tends to the
minimax polynomial.  With n = 513 and 100 iterations the coefficients
agree with sm100.cuh's to all printed digits, max relative error 7.48e-5.

Run: python fit_exp2_poly.py  (prints c0..c3 and the max relative error)."""
import numpy as np


def fit(deg: int = 3, n: int = 513, iters: int = 100) -> np.ndarray:
    k = np.arange(n)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / n)
    y = np.exp2(f)
    V = np.vander(f, deg + 1, increasing=True)
    w = np.full(n, 1.0 / n)
    c = np.zeros(deg + 1)
    for _ in range(iters):
        W = np.sqrt(w) / y
        c, *_ = np.linalg.lstsq(V * W[:, None], y * W, rcond=None)
        e = np.abs(V @ c - y) / y
        w = w * e
        w /= w.sum()
    return c  # c[0] + c[1] f + c[2] f^2 + c[3] f^3


def max_rel_error(c, m: int = 200001) -> float:
    f = np.linspace(-0.5, 0.5, m)
    return float(np.max(np.abs(np.polyval(np.asarray(c)[::-1], f) - np.exp2(f)) / np.exp2(f)))


if __name__ == "__main__":
    c = fit()
    print("coefficients c0..c3:", ", ".join(f"{x:.8g}" for x in c))
    print("max relative error on [-1/2, 1/2]:", f"{max_rel_error(c):.3e}")
