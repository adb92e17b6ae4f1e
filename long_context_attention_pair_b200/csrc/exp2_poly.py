"""Coefficients of the polynomial 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on f in [-1/2, 1/2].

Used by the prefill kernel for the share of softmax exponentials it evaluates on
the FMA pipe instead of the multi-function unit (Cody-Waite range reduction:
x = n + f with n = round(x), 2^x = 2^n * 2^f).  Fit: least squares on Chebyshev
nodes of the first kind, weighted by 1/2^f so that the RELATIVE error is
minimised, then the constant term is adjusted so the fit is exact at f = 0
(2^0 = 1, so p = 1 and exp2 of an exact integer is exact).

Run:  python exp2_poly.py   (prints the coefficients and the max relative error
in float32 Horner evaluation; the values are pasted into prefill_tc.cu).
"""
import numpy as np

DEGREE = 3


def fit(degree=DEGREE, nodes=4001):
    k = np.arange(nodes)
    f = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * nodes))  # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]
    c, *_ = np.linalg.lstsq(A, np.ones_like(f), rcond=None)
    c[0] = 1.0
    return c


def horner_f32(c, f):
    f = f.astype(np.float32)
    c = c.astype(np.float32)
    p = np.full_like(f, c[-1])
    for ci in c[-2::-1]:
        p = (p * f + ci).astype(np.float32)
    return p


def max_rel_error(c, samples=200001):
    f = np.linspace(-0.5, 0.5, samples)
    p = horner_f32(c, f).astype(np.float64)
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit()
    print("coefficients (float32):", ", ".join(f"{np.float32(x)!r}" for x in c))
    print("max relative error (float32 Horner): %.3e" % max_rel_error(c))
