"""Derive the polynomial constants used by the scan kernels' pointwise math.

    python selective_state_space_ss_b200/csrc/fit_poly.py

Prints C initialisers.  Each fit is a weighted least-squares polynomial on a
dense grid (Chebyshev-distributed nodes), solved in float64, then the
coefficients are rounded to float32 and the worst error of the float32 Horner
evaluation is reported.  The constants in pointwise.cuh are this script's
output; tests/test_pointwise_fits.py re-runs the fits, checks them against the header
and evaluates every function on the device against float64.

Fits
  log1p_over:  log1p(e) / e  on e in [0, 1]        (softplus = max(x,0) + log1p(e^-|x|))
  exp2_frac:   2^f           on f in [-0.5, 0.5]   (2^x = 2^k * 2^f, k = round(x))
"""
from __future__ import annotations

import numpy as np


def _cheb_nodes(a, b, n):
    k = np.arange(n)
    return 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * (k + 0.5) / n)


def fit(func, a, b, degree, rel=True, n=4000):
    x = _cheb_nodes(a, b, n)
    y = func(x)
    w = 1.0 / np.abs(y) if rel else np.ones_like(y)
    V = np.vander(x, degree + 1, increasing=True)
    c, *_ = np.linalg.lstsq(V * w[:, None], y * w, rcond=None)
    return c


def horner_f32(c, x):
    x = x.astype(np.float32)
    acc = np.float32(c[-1]) * np.ones_like(x)
    for ci in c[-2::-1]:
        acc = (acc * x + np.float32(ci)).astype(np.float32)
    return acc


def log1p_over_coeffs(degree=8):
    f = lambda e: np.where(e == 0, 1.0, np.log1p(e) / np.where(e == 0, 1.0, e))
    return np.float32(fit(f, 0.0, 1.0, degree))


def exp2_frac_coeffs(degree=6):
    return np.float32(fit(lambda t: np.exp2(t), -0.5, 0.5, degree))


def max_rel_err(c, func, a, b, n=200001):
    x = np.linspace(a, b, n, dtype=np.float64).astype(np.float32)
    got = horner_f32(c, x).astype(np.float64)
    ref = func(x.astype(np.float64))
    return float(np.max(np.abs(got - ref) / np.abs(ref)))


def main():
    lp = log1p_over_coeffs()
    e2 = exp2_frac_coeffs()
    f_lp = lambda e: np.where(e == 0, 1.0, np.log1p(e) / np.where(e == 0, 1.0, e))
    print("// log1p(e)/e on [0,1], degree", len(lp) - 1, "max rel err",
          f"{max_rel_err(lp, f_lp, 0.0, 1.0):.2e}")
    print("{" + ", ".join(f"{v:.9e}f" for v in lp) + "}")
    print("// 2^f on [-0.5,0.5], degree", len(e2) - 1, "max rel err",
          f"{max_rel_err(e2, np.exp2, -0.5, 0.5):.2e}")
    print("{" + ", ".join(f"{v:.9e}f" for v in e2) + "}")


if __name__ == "__main__":
    main()
