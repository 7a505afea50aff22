"""Fit of the polynomial the prefill softmax uses for part of its 2^x.

The softmax evaluates some of its exponentials on the FMA pipes instead of
the special-function unit: 2^x = 2^n * 2^f with n = x rounded to the nearest
integer and f = x - n in [-0.5, 0.5] (Cody and Waite's range reduction), and
2^f approximated by a cubic p(f) = 1 + c1 f + c2 f^2 + c3 f^3.

The coefficients below are the minimax fit of the relative error
|p(f) / 2^f - 1| over [-0.5, 0.5] with p(0) = 1, solved as a linear program
on a dense grid, then rounded to fp32. Re-running this module reproduces them
and reports the error of the fp32 Horner evaluation (about 1.0e-4, far below
the 2^-9 half-ulp of the bf16 the probabilities are rounded to).

    python -m ragged_paged_kv_rope_b200.exp2_poly_fit
"""

from __future__ import annotations

import numpy as np

# The values compiled into csrc/attn_prefill.cu (kExp2C1..kExp2C3).
COEFFS = (1.0, 0.6932829022407532, 0.2422109693288803, 0.055009059607982635)


def fit(degree: int = 3, points: int = 4001):
    from scipy.optimize import linprog

    f = np.linspace(-0.5, 0.5, points)
    y = np.exp2(f)
    A = np.stack([f ** k / y for k in range(1, degree + 1)], axis=1)
    b0 = 1.0 / y - 1.0
    ones = np.ones((points, 1))
    a_ub = np.vstack([np.hstack([A, -ones]), np.hstack([-A, -ones])])
    b_ub = np.concatenate([-b0, b0])
    res = linprog(np.r_[np.zeros(degree), 1.0], A_ub=a_ub, b_ub=b_ub,
                  bounds=[(None, None)] * degree + [(0, None)])
    if not res.success:
        raise RuntimeError(res.message)
    return tuple(float(np.float32(c)) for c in np.r_[1.0, res.x[:degree]])


def max_rel_error(coeffs, points: int = 100001) -> float:
    """Max relative error of the fp32 Horner evaluation of p(f) against 2^f."""
    f = np.linspace(-0.5, 0.5, points).astype(np.float32)
    c = [np.float32(x) for x in coeffs]
    p = np.float32(c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = p * f + c[k]
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = fit()
    print("coefficients", c)
    print("max relative error (fp32 Horner)", max_rel_error(c))
