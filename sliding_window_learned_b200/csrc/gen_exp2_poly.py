"""Writes exp2_poly.h: the polynomial the forward kernel uses to evaluate part
of its 2^x terms on the FMA pipe instead of the MUFU unit.

Method (Cody and Waite's argument reduction): write x = n + f with
n = round(x) and f in [-1/2, 1/2], so that 2^x = 2^n * 2^f; 2^n is applied by
adding n to the float's exponent field, and 2^f is approximated by a
polynomial p(f) of degree 3.  The coefficients here are a weighted least-
squares fit of 2^f on 2049 Chebyshev nodes of [-1/2, 1/2] with weight 2^-f
(i.e. minimising the relative error), rounded to float32.

The kernel rounds each probability to bf16 (relative spacing 2^-8) before the
P.V product, so a relative error near 1e-4 is far below that rounding.  The
script prints the measured maximum relative error of the float32 evaluation.

Usage: python gen_exp2_poly.py   (rewrites exp2_poly.h next to this file)
"""
import os

import numpy as np

DEGREE = 3


def fit(degree: int) -> np.ndarray:
    k = np.arange(2049)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / len(k))          # Chebyshev nodes in [-1/2, 1/2]
    target = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / target[:, None]
    coef, *_ = np.linalg.lstsq(A, np.ones_like(f), rcond=None)
    return coef.astype(np.float32)


def max_rel_error(coef: np.ndarray) -> float:
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    acc = np.full_like(f, coef[-1])
    for c in coef[-2::-1]:                                 # Horner in float32
        acc = (acc * f + np.float32(c)).astype(np.float32)
    return float(np.max(np.abs(acc.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1)))


def main():
    coef = fit(DEGREE)
    err = max_rel_error(coef)
    here = os.path.dirname(os.path.abspath(__file__))
    lines = [
        "// exp2_poly.h -- written by gen_exp2_poly.py; do not edit.",
        "// 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on f in [-1/2, 1/2]: weighted least-squares",
        "// fit on Chebyshev nodes (relative error), after Cody-Waite reduction x = n + f.",
        f"// measured max relative error (float32 Horner): {err:.3e}",
        "#pragma once",
        "namespace attnsink {",
    ]
    for i, c in enumerate(coef):
        lines.append(f"constexpr float kExp2C{i} = {float(c)!r}f;")
    lines += [f"constexpr float kExp2PolyMaxRelErr = {err:.3e}f;", "}  // namespace attnsink", ""]
    with open(os.path.join(here, "exp2_poly.h"), "w") as fh:
        fh.write("\n".join(lines))
    print(f"degree {DEGREE}: coefficients {coef.tolist()} max rel err {err:.3e}")


if __name__ == "__main__":
    main()
