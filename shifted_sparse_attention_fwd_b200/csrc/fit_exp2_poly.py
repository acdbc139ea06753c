"""Coefficients of the cubic for 2^f on [-0.5, 0.5] used by exp2_poly2 (s2_device.cuh).

Least squares on 4001 Chebyshev nodes, each residual weighted by 1 / 2^f so that the fit
minimises relative error. Prints the float32 coefficients and the maximum relative error of
the float32 polynomial on a fine grid.
"""
import numpy as np


def fit(degree: int = 3):
    x = 0.5 * np.cos(np.linspace(0.0, np.pi, 4001))
    w = 1.0 / 2.0 ** x
    a = np.vander(x, degree + 1, increasing=True)
    c, *_ = np.linalg.lstsq(a * w[:, None], 2.0 ** x * w, rcond=None)
    return c.astype(np.float32)


def max_rel_err(c) -> float:
    f = np.linspace(-0.5, 0.5, 200001)
    p = np.polyval(np.asarray(c, dtype=np.float64)[::-1], f)
    return float(np.max(np.abs(p / 2.0 ** f - 1.0)))


if __name__ == "__main__":
    c = fit()
    print("coefficients c0..c3:", ", ".join(f"{v!r}" for v in c.tolist()))
    print("max relative error:", max_rel_err(c))
