"""Fit the polynomial the attention kernel uses for 2^f on f in [-1/2, 1/2].

The kernel evaluates part of its exponentials on the FMA pipe instead of the
special-function unit:

    2^x = 2^j * 2^f,   j = round(x) (integer),   f = x - j in [-1/2, 1/2]

j is obtained by adding and subtracting 1.5 * 2^23 (round-to-nearest in
fp32), 2^f by a polynomial, and 2^j by adding j to the exponent field of the
result.  This script derives the polynomial: a minimax fit of the *relative*
error by Lawson's iteratively reweighted least squares on a dense grid, with
the constant term fixed to 1 so that 2^0 = 1 exactly.  It prints the
coefficients (rounded to fp32) and the maximum relative error of the fp32
Horner evaluation.

Run: python exact_tiled_attention_45_b200/csrc/fit_exp2_poly.py [degree]
"""
from __future__ import annotations

import sys

import numpy as np


def fit(degree: int, iters: int = 400, n: int = 20001):
    f = np.linspace(-0.5, 0.5, n)
    target = np.exp2(f)
    # p(f) = 1 + sum_{k=1..deg} c_k f^k ; minimise max |p/target - 1|
    A = np.stack([f ** k for k in range(1, degree + 1)], axis=1) / target[:, None]
    b = 1.0 - 1.0 / target
    w = np.ones(n) / n
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    return np.concatenate([[1.0], c])


def horner_fp32(coef32: np.ndarray, f: np.ndarray) -> np.ndarray:
    f = f.astype(np.float32)
    acc = np.full_like(f, coef32[-1])
    for c in coef32[-2::-1]:
        acc = (acc * f + c).astype(np.float32)  # the kernel uses fused multiply-add
    return acc


def max_rel_error(coef32: np.ndarray) -> float:
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    approx = horner_fp32(coef32, f).astype(np.float64)
    return float(np.max(np.abs(approx / np.exp2(f.astype(np.float64)) - 1.0)))


def main():
    degree = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    coef = fit(degree)
    coef32 = coef.astype(np.float32)
    for k, c in enumerate(coef32):
        print(f"c{k} = {float(c)!r}  ({np.float32(c).view(np.uint32):#010x})")
    print(f"max relative error (fp32 Horner on [-1/2, 1/2]): {max_rel_error(coef32):.3e}")


if __name__ == "__main__":
    main()
