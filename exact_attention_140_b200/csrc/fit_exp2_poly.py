"""Derivation of the software exp2 polynomial used by the attention kernel.

2^x is split as 2^j * 2^f with j = round(x) and f = x - j in [-0.5, 0.5].
2^f is approximated by p(f) = 1 + c1 f + c2 f^2 + c3 f^3 (p(0) = 1 exactly,
so 2^0 is exact), with c1..c3 chosen to minimise the maximum relative error
max |p(f)/2^f - 1| over [-0.5, 0.5]: a linear program on a dense grid.  The
coefficients are then rounded to fp32 and the error re-measured with fp32
Horner evaluation.  Run: python fit_exp2_poly.py
"""
import numpy as np
from scipy.optimize import linprog


def fit(n_grid: int = 20001):
    f = np.linspace(-0.5, 0.5, n_grid)
    y = 2.0 ** f
    A = np.stack([f, f ** 2, f ** 3], 1)
    A_ub = np.vstack([np.hstack([A, -y[:, None]]), np.hstack([-A, -y[:, None]])])
    b_ub = np.concatenate([y - 1.0, 1.0 - y])
    res = linprog([0, 0, 0, 1], A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * 3 + [(0, None)])
    assert res.status == 0
    return res.x[:3], res.x[3]


def fp32_error(c):
    c = np.asarray(c, dtype=np.float32)
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = c[2]
    p = p * f + c[1]
    p = p * f + c[0]
    p = p * f + np.float32(1.0)
    return float(np.max(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0)))


if __name__ == "__main__":
    c, err = fit()
    c32 = np.asarray(c, dtype=np.float32)
    print("c1, c2, c3 =", ", ".join(f"{x:.9g}f" for x in c32))
    print(f"minimax relative error (fp64) = {err:.3e} (2^{np.log2(err):.2f})")
    print(f"with fp32 coefficients and fp32 Horner = {fp32_error(c32):.3e}")
