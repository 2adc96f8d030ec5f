"""Fit the polynomial used by the softmax kernels to evaluate 2^f on the FMA pipe.

Method (Lawson's iteratively re-weighted least squares, which converges to the minimax
approximation): minimise the maximum RELATIVE error of a degree-4 polynomial p(f) to
2^f on f in [-0.5, 0.5]. The kernel reduces x = j + f with j = round-to-nearest(x), so
|f| <= 1/2, evaluates p(f) with fused multiply-adds (Horner), and adds j to the float's
exponent field. Coefficients are rounded to fp32; the script reports the relative error
of the fp32 Horner evaluation on a dense grid.

Usage: python io_aware_exact_28_b200/csrc/fit_exp2_poly.py   (prints the C constants)
"""
from __future__ import annotations

import numpy as np

DEGREE = 4


def fit(degree: int = DEGREE, iters: int = 200, npts: int = 4001):
    f = np.cos(np.linspace(0.0, np.pi, npts)) * 0.5          # Chebyshev-distributed nodes
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)
    w = np.ones_like(f)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w) / y                                 # relative error weighting
        c, *_ = np.linalg.lstsq(V * sw[:, None], y * sw, rcond=None)
        err = np.abs(V @ c - y) / y
        w = w * err
        w /= w.sum()
    return c


def horner_f32(c32: np.ndarray, f: np.ndarray) -> np.ndarray:
    p = np.full_like(f, c32[-1], dtype=np.float32)
    for a in c32[-2::-1]:
        p = (p.astype(np.float64) * f + a).astype(np.float32)   # one rounding per FMA
    return p


def max_rel_error(c32: np.ndarray) -> float:
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    return float(np.max(np.abs(horner_f32(c32, f).astype(np.float64) - np.exp2(f.astype(np.float64)))
                        / np.exp2(f.astype(np.float64))))


def main():
    c = fit()
    c32 = c.astype(np.float32)
    print(f"// degree {DEGREE}, max relative error of fp32 Horner on [-0.5, 0.5]: {max_rel_error(c32):.3e}")
    for i, a in enumerate(c32):
        print(f"constexpr float kExp2C{i} = {float(a).hex()}f;  // {float(a):.9g}")


if __name__ == "__main__":
    main()
