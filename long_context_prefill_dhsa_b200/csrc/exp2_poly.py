"""Coefficients of the polynomial 2^f used for part of the softmax exponentials.

The attention kernel evaluates some of its exponentials 2^x on the FMA pipe
instead of the special-function unit: x = j + f with j = round(x) and
|f| <= 1/2, 2^j goes into the exponent field, and 2^f comes from

    q(f) = 1 + f * (c1 + f * (c2 + f * c3)).

The constant term is fixed at 1 so that x = 0 (the score at the running row
maximum) gives exactly 1. c1..c3 minimise the maximum relative error
|q(f) / 2^f - 1| over [-1/2, 1/2], posed as a linear program on a dense grid.

Run `python exp2_poly.py` to print the coefficients, rounded to fp32, and the
relative error of the fp32 evaluation (magic-constant rounding, FMA Horner
steps, exponent add) over [-126, 8]; below -126 the kernel's clamp at -127
gives values in [0, 2^-126), exactly 0 from -127 down.
"""
import numpy as np
from scipy.optimize import linprog


def fit(degree=3, points=8193):
    """c1..c_degree and the minimax relative error E."""
    f = np.linspace(-0.5, 0.5, points)
    y = np.exp2(f)
    # |1 + A c - y| / y <= E with A[:, i] = f^(i+1): two one-sided rows per point
    A = np.vstack([f ** i / y for i in range(1, degree + 1)]).T
    ones = np.ones((points, 1))
    A_ub = np.vstack([np.hstack([A, -ones]), np.hstack([-A, -ones])])
    b_ub = np.concatenate([1.0 - 1.0 / y, 1.0 / y - 1.0])
    cost = np.zeros(degree + 1)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * (degree + 1), method="highs")
    if not res.success:
        raise RuntimeError(res.message)
    return res.x[:-1].astype(np.float32), float(res.x[-1])


def _fma32(a, b, d):
    """fp32 fused multiply-add: the exact product-sum, rounded once (fp64 holds it
    exactly for these magnitudes except in rare double-rounding cases)."""
    return (np.float64(a) * np.asarray(b, np.float64) + np.float64(d)).astype(np.float32)


def exp2_fp32(x, c):
    """The kernel's fp32 steps, each rounded to fp32."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-127.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)   # 1.5 * 2^23
    j = (t - np.float32(12582912.0)).astype(np.float32)
    fr = (x.astype(np.float64) - j.astype(np.float64)).astype(np.float32)
    q = _fma32(c[2], fr, c[1])
    q = (q.astype(np.float64) * fr + np.float64(c[0])).astype(np.float32)
    q = (q.astype(np.float64) * fr + 1.0).astype(np.float32)
    bits = q.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def main():
    c, e = fit()
    print("c1, c2, c3 =", ", ".join(f"{v:.8f}f" for v in c))
    print(f"minimax relative error of the polynomial: {e:.3e}")
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-126, 8, 1_000_000), np.linspace(-3, 3, 100_001)]).astype(np.float32)
    rel = np.abs(exp2_fp32(x, c) / np.exp2(x.astype(np.float64)) - 1.0)
    print(f"fp32 evaluation over [-126, 8]: max relative error {rel.max():.3e}")


if __name__ == "__main__":
    main()
