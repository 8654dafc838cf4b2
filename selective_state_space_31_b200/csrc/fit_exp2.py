"""Derive the polynomial of the kernels' FMA-pipe 2^x (device_common.cuh,
``exp2_fma2``).

Method (range reduction in the style of Cody and Waite): x = n + f with n the
integer nearest x and f in [-1/2, 1/2]; 2^x = 2^n * 2^f, the power of two
formed by adding n to the exponent field.  2^f is written 1 + f * Q(f), so
f = 0 gives exactly 1, and Q approximates (2^f - 1) / f: a least-squares fit
in the Chebyshev basis on 4000 Chebyshev nodes of [-1/2, 1/2], weighted by
f / 2^f so that the residual is the relative error of 2^f (near minimax),
converted to monomial coefficients and rounded to float32.  Prints the
coefficients and the maximum relative error of the float32 Horner evaluation
against numpy's float64 2^f on a dense grid.

    python selective_state_space_31_b200/csrc/fit_exp2.py [degree of Q]
"""
import sys

import numpy as np


def fit(deg: int):
    n = 4000
    f = np.cos(np.pi * (np.arange(n) + 0.5) / n) * 0.5
    q = np.expm1(f * np.log(2.0)) / f
    w = np.abs(f) / np.exp2(f)
    c = np.polynomial.chebyshev.chebfit(2 * f, q, deg, w=w)   # basis variable 2f in [-1, 1]
    p = np.polynomial.Polynomial(np.polynomial.chebyshev.cheb2poly(c))
    mono = p(np.polynomial.Polynomial([0.0, 2.0]))             # substitute u = 2f
    return mono.coef.astype(np.float32)


def evaluate(coef, f):
    acc = np.full_like(f, coef[-1])
    for k in range(len(coef) - 2, -1, -1):
        acc = (acc * f + coef[k]).astype(np.float32)
    return (acc * f + np.float32(1.0)).astype(np.float32)


def max_rel_error(coef):
    fg = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    val = evaluate(coef, fg).astype(np.float64)
    ref = np.exp2(fg.astype(np.float64))
    return float(np.max(np.abs(val - ref) / ref))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    coef = fit(deg)
    print("coefficients of Q (f^0 .. f^%d):" % deg)
    for k, v in enumerate(coef):
        print(f"  q{k} = {float(v):.9g}f")
    print(f"max relative error of 1 + f*Q(f) (float32 Horner): {max_rel_error(coef):.3e}")
