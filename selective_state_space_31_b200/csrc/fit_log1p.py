"""Derive the polynomial used for log1p(u), u in [0, 1], in the kernels'
softplus (device_common.cuh, ``log1p_unit``).

Method: least-squares fit of f(u) = log1p(u) / u in the Chebyshev basis on
4000 Chebyshev nodes of [0, 1] (a near-minimax approximation), converted to
monomial coefficients in u and rounded to float32; log1p(u) is then
u * P(u) evaluated by Horner's rule in float32.  Prints the coefficients and
the maximum relative error of that float32 evaluation against numpy's
float64 log1p on a dense grid.

    python selective_state_space_31_b200/csrc/fit_log1p.py [degree]
"""
import sys

import numpy as np


def fit(deg: int):
    n = 4000
    u = np.cos(np.pi * (np.arange(n) + 0.5) / n) * 0.5 + 0.5
    c = np.polynomial.chebyshev.chebfit(2 * u - 1, np.log1p(u) / u, deg)
    p = np.polynomial.Polynomial(np.polynomial.chebyshev.cheb2poly(c))
    mono = p(np.polynomial.Polynomial([-1.0, 2.0]))       # substitute x = 2u - 1
    return mono.coef.astype(np.float32)


def max_rel_error(coef):
    ug = np.linspace(0, 1, 400001).astype(np.float32)[1:]
    acc = np.full_like(ug, coef[-1])
    for k in range(len(coef) - 2, -1, -1):
        acc = (acc * ug + coef[k]).astype(np.float32)
    val = (acc * ug).astype(np.float64)
    ref = np.log1p(ug.astype(np.float64))
    return float(np.max(np.abs(val - ref) / ref))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 8
    coef = fit(deg)
    print("coefficients (u^0 .. u^%d):" % deg)
    for k, v in enumerate(coef):
        print(f"  c{k} = {float(v):.9g}f")
    print(f"max relative error (float32 Horner): {max_rel_error(coef):.3e}")
