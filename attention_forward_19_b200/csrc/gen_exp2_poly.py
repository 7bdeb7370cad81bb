"""Fits the polynomial used by the kernel's FMA-pipe exp2.

The kernel computes 2^x for part of the softmax elements without the MUFU
unit: x = j + r with j = round(x) (an integer) and r in [-1/2, 1/2], then
2^x = 2^j * 2^r where 2^j is added to the float's exponent field and 2^r is a
polynomial.  This script fits that polynomial: near-minimax in relative error
on [-1/2, 1/2] (Lawson's iteratively reweighted least squares on a dense
grid), with the constant term fixed to 1 so that 2^0 is exact.  The printed
coefficients are rounded to fp32 and the resulting relative error is checked
in fp32 arithmetic (Horner with fused multiply-adds).

    python attention_forward_19_b200/csrc/gen_exp2_poly.py
"""
import numpy as np


def fit(degree, iters=400):
    r = np.linspace(-0.5, 0.5, 20001)
    f = np.exp2(r)
    # unknowns c1..cd of p(r) = 1 + c1 r + ... + cd r^d; relative residual (p - f) / f
    A = np.stack([r ** k / f for k in range(1, degree + 1)], axis=1)
    b = (f - 1.0) / f
    w = np.ones_like(r) / len(r)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    coeffs = np.concatenate([[1.0], c]).astype(np.float32)
    return coeffs


def rel_error_fp32(coeffs):
    r = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    acc = np.float32(coeffs[-1]) * np.ones_like(r)
    for c in coeffs[-2::-1]:
        acc = (acc.astype(np.float64) * r + np.float64(c)).astype(np.float32)   # fma rounding
    exact = np.exp2(r.astype(np.float64))
    return float(np.max(np.abs(acc / exact - 1.0)))


if __name__ == "__main__":
    for deg in (3, 4, 5):
        c = fit(deg)
        print(f"degree {deg}: coefficients c0..c{deg} =",
              ", ".join(f"{float(x):.9e}f" for x in c), f"; max rel error {rel_error_fp32(c):.3e}")
