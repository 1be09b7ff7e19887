"""Generates the coefficients of the polynomial p with log1p(u) ~ u p(u) on
[0, 1] that the decay steps (csrc/ssd_math.cuh, softplus_fast) use: Chebyshev
interpolation of log1p(u)/u at the degree + 1 Chebyshev nodes of [0, 1],
converted to powers of u and rounded to float32.  Prints the coefficients
(constant term first) and the largest relative error of u p(u) against
log1p(u) over [1e-12, 1], evaluated by float32 Horner steps.

    python -m mamba_ssd_sequence_b200.gen_log1p_poly [degree]
"""
import sys

import numpy as np


def coefficients(degree: int = 8) -> np.ndarray:
    k = np.arange(degree + 1)
    t = np.cos((2 * k + 1) * np.pi / (2 * (degree + 1)))  # nodes on [-1, 1]
    u = (t + 1) / 2
    cheb = np.polynomial.chebyshev.chebfit(t, np.log1p(u) / u, degree)
    poly = np.polynomial.Chebyshev(cheb, domain=[0, 1]).convert(kind=np.polynomial.Polynomial)
    return poly.coef.astype(np.float32)


def max_rel_error(c32: np.ndarray) -> float:
    u = np.linspace(1e-12, 1.0, 2_000_001)
    x = u.astype(np.float32)
    acc = np.full_like(x, c32[-1])
    for c in c32[-2::-1]:
        acc = (acc * x + c).astype(np.float32)
    return float(np.max(np.abs((x * acc).astype(np.float64) - np.log1p(u)) / np.log1p(u)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 8
    c = coefficients(deg)
    print(", ".join(f"{v:.9e}f" for v in c))
    print("max relative error:", max_rel_error(c))
