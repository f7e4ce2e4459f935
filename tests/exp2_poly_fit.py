"""Fit the polynomial used by the attention kernel's software 2^x.

Method: 2^x = 2^n * 2^f with n = rint(x) and f = x - n in [-1/2, 1/2] (Cody-Waite style
range reduction with a single constant, exact here because n is an integer); 2^f is
approximated by a degree-3 polynomial whose coefficients minimise the maximum relative
error over [-1/2, 1/2].  The minimax problem is solved on a dense grid as a linear
program (minimise t subject to |p(f_i) - 2^f_i| <= t * 2^f_i), then the coefficients are
rounded to float32 and the error of the float32 Horner evaluation is measured.

Run ``python -m tests.exp2_poly_fit`` to print the
coefficients written into ``attn_fwd_sm100.cuh`` (kExp2C0..kExp2C3).
"""

from __future__ import annotations

import numpy as np

DEGREE = 3


def fit(degree: int = DEGREE, n_grid: int = 4001):
    from scipy.optimize import linprog

    f = np.linspace(-0.5, 0.5, n_grid)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)  # columns f^0 .. f^degree
    # variables: c_0..c_degree, t ; minimise t
    nvar = degree + 2
    cost = np.zeros(nvar)
    cost[-1] = 1.0
    A = np.vstack([np.hstack([V, -y[:, None]]), np.hstack([-V, -y[:, None]])])
    b = np.concatenate([y, -y])
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * nvar, method="highs")
    assert res.success, res.message
    return res.x[:-1], res.x[-1]


def float32_error(coef) -> float:
    """Max relative error of the float32 Horner evaluation p(f) on a dense grid of [-1/2, 1/2]."""
    c = np.asarray(coef, dtype=np.float32)
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + c[k]).astype(np.float32)  # Horner, one rounding per step (an FMA rounds once)
    ref = np.exp2(f.astype(np.float64))
    return float(np.max(np.abs(p.astype(np.float64) - ref) / ref))


def coefficients():
    c, _ = fit()
    return [float(np.float32(x)) for x in c]


if __name__ == "__main__":
    c, t = fit()
    c32 = [np.float32(x) for x in c]
    print(f"degree {DEGREE}: minimax relative error {t:.3e}; float32 Horner error {float32_error(c32):.3e}")
    for i, x in enumerate(c32):
        print(f"constexpr float kExp2C{i} = {float(x)!r}f;  // {np.float32(x).view(np.uint32):#010x}")
