"""Fit the polynomial the kernels use for log1p on [0, 1].

softplus(t) = max(t, 0) + log1p(z), z = exp(-|t|) in (0, 1].  The kernels
evaluate log1p(z) = z * q(z) where q approximates log1p(z) / z on [0, 1] (a
smooth function, from 1 at z = 0 to ln 2 at z = 1).  q is a degree-7
Chebyshev least-squares fit (4000 Chebyshev nodes on [0, 1]), converted to the
monomial basis for Horner evaluation; this script prints the coefficients and
the worst relative error of z * q(z) against log1p(z) when q is evaluated in
fp32 with Horner's rule on a dense grid.  The constants in common.cuh are the
output of this script.

    python selective_scan_crossscan_b200/csrc/fit_softplus_poly.py
"""
import numpy as np

DEGREE = 7


def fit(degree: int = DEGREE):
    m = 4000
    z = np.cos(np.pi * (np.arange(m) + 0.5) / m) * 0.5 + 0.5  # Chebyshev nodes on [0, 1]
    q = np.log1p(z) / z
    cheb = np.polynomial.chebyshev.chebfit(2.0 * z - 1.0, q, degree)
    in_x = np.polynomial.chebyshev.cheb2poly(cheb)  # monomials in x = 2z - 1
    in_z = np.polynomial.Polynomial(in_x)(np.polynomial.Polynomial([-1.0, 2.0]))  # substitute x = 2z - 1
    return in_z.coef


def worst_relative_error(coef) -> float:
    c32 = np.asarray(coef, dtype=np.float32)
    z = np.linspace(0.0, 1.0, 400001).astype(np.float32)[1:]
    acc = np.full_like(z, c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        acc = (acc * z + c32[k]).astype(np.float32)
    approx = (z * acc).astype(np.float64)
    exact = np.log1p(z.astype(np.float64))
    return float(np.max(np.abs(approx - exact) / exact))


if __name__ == "__main__":
    coef = fit()
    for k, c in enumerate(coef):
        print(f"c{k} = {np.float32(c)!r}  ({c:.17g})")
    print(f"max relative error of z*q(z) vs log1p(z), fp32 Horner: {worst_relative_error(coef):.3e}")
