"""Fit the polynomial the attention kernel uses for part of its exp2 evaluations.

The kernel computes 2^x for x <= 0 as 2^j * q(f) with j = round(x) (a magic-number add) and
f = x - j in [-0.5, 0.5]; q approximates 2^f. This script derives q by minimising the maximum
*relative* error on [-0.5, 0.5] with a Lawson-weighted least-squares iteration (each pass
reweights the sample points by their error so the solution converges to the equioscillating
minimax fit), then rounds the coefficients to float32 and reports the error of the rounded
polynomial evaluated in float32 Horner form.

    python -m precision_attention_forward_b200.csrc.exp2_poly_fit [degree]

The printed coefficients are the ones in attn_fwd.cuh (kExp2Poly*).
"""
from __future__ import annotations

import sys

import numpy as np


def fit(degree: int, points: int = 4001, iters: int = 400):
    f = np.cos(np.linspace(0.0, np.pi, points)) * 0.5          # Chebyshev-spaced on [-0.5, 0.5]
    target = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / target[:, None]   # relative error rows
    b = np.ones_like(f)
    w = np.full(points, 1.0 / points)
    coef = None
    for _ in range(iters):
        sw = np.sqrt(w)
        coef, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ coef - b)
        w = w * err
        w /= w.sum()
    return coef


def rounded_error(coef32: np.ndarray, samples: int = 200001) -> float:
    f = np.linspace(-0.5, 0.5, samples).astype(np.float32)
    acc = np.full_like(f, coef32[-1])
    for c in coef32[-2::-1]:
        acc = (acc * f + np.float32(c)).astype(np.float32)
    return float(np.max(np.abs(acc.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


def main():
    degree = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    coef = fit(degree)
    c32 = coef.astype(np.float32)
    for i, c in enumerate(c32):
        print(f"c{i} = {float(c)!r:>24}  ({float(c).hex()})")
    print(f"max relative error in float32 Horner evaluation: {rounded_error(c32):.3e}")


if __name__ == "__main__":
    main()
