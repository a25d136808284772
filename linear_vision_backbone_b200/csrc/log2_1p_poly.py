"""Coefficients of the polynomial the kernels use for log2(1 + t), t in [0, 1].

Method: Chebyshev interpolation (the interpolant through the 9 Chebyshev
nodes of the first kind, x_k = cos(pi (k + 1/2) / 9), mapped to t = (x + 1) / 2)
of q(t) = log2(1 + t) / t, a function analytic on [0, 1] with q(0) = 1 / ln 2,
rewritten in powers of t for Horner evaluation; log2(1 + t) = t q(t) is then
exactly 0 at t = 0 and positive for t > 0.  Printed as the fp32 constants of
tc_kernels.cuh (kL2q); with fp32 Horner evaluation the absolute error of
t q(t) on [0, 1] is below 1.6e-7 (checked here on a dense grid).

    python log2_1p_poly.py
"""
import numpy as np
from numpy.polynomial import chebyshev as C
from numpy.polynomial import polynomial as P

DEG = 8


def q(t):
    t = np.asarray(t, dtype=np.float64)
    safe = np.where(t > 0, t, 1.0)
    return np.where(t > 0, np.log2(1.0 + safe) / safe, 1.0 / np.log(2.0))


def coefficients(deg=DEG):
    x = np.cos(np.pi * (np.arange(deg + 1) + 0.5) / (deg + 1))
    c = C.chebfit(x, q((x + 1.0) / 2.0), deg)     # interpolation: deg + 1 nodes, degree deg
    px = C.cheb2poly(c)                           # powers of x
    pt = np.zeros(1)
    for a in px[::-1]:                            # x = 2 t - 1, Horner in t
        pt = P.polyadd(P.polymul(pt, [-1.0, 2.0]), [a])
    return pt.astype(np.float32)


def max_error(coef):
    t = np.linspace(0.0, 1.0, 1 << 20).astype(np.float32)
    acc = np.float32(coef[-1]) * np.ones_like(t)
    for a in coef[-2::-1]:
        acc = (acc * t + np.float32(a)).astype(np.float32)
    val = (acc * t).astype(np.float32)
    return float(np.abs(val.astype(np.float64) - np.log2(1.0 + t.astype(np.float64))).max())


if __name__ == "__main__":
    coef = coefficients()
    print("max |t q(t) - log2(1 + t)| =", max_error(coef))
    print("{" + ", ".join(f"{float(a):.9e}f" for a in coef) + "}")
