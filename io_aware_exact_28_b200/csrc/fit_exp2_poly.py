"""Fit the polynomial that exp2_emu (sm100.cuh) uses to evaluate 2^x on the FMA pipe.

The kernel splits x = j + f with j = round-to-nearest(x) (the 1.5 * 2^23 shifter), so
|f| <= 1/2, evaluates p(f) = 1 + f (c1 + f (c2 + f (c3 + f c4))) with four fused
multiply-adds, and adds j to the result's exponent field. The constant term is pinned to
exactly 1, so that p(0) = 1 and the clamp of x at -127 (masked keys, x = -inf) gives the
bit pattern of 1.0 minus 127 << 23, which is +0 exactly.

Method: Lawson's iteratively re-weighted least squares, which converges to the minimax
fit, on the maximum RELATIVE error |p(f) - 2^f| / 2^f over Chebyshev-distributed nodes
of [-1/2, 1/2]. Coefficients are rounded to fp32; max_rel_error reports the error of the
fp32 Horner evaluation on a dense grid.

Usage: python io_aware_exact_28_b200/csrc/fit_exp2_poly.py   (prints the C constants)
"""
from __future__ import annotations

import numpy as np

DEGREE = 4


def fit(degree: int = DEGREE, iters: int = 300, npts: int = 4001) -> np.ndarray:
    """Coefficients [1, c1, ..., c_degree] (float64) of p(f) ~ 2^f on [-1/2, 1/2]."""
    f = np.cos(np.linspace(0.0, np.pi, npts)) * 0.5
    y = np.exp2(f)
    # p(f) - 1 = f * sum_k c_k f^(k-1): columns f^1 .. f^degree, target 2^f - 1.
    V = np.vander(f, degree + 1, increasing=True)[:, 1:]
    w = np.ones_like(f)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w) / y                         # relative error weighting
        c, *_ = np.linalg.lstsq(V * sw[:, None], (y - 1.0) * sw, rcond=None)
        err = np.abs(1.0 + V @ c - y) / y
        w = w * (err + 1e-300)
        w /= w.sum()
    return np.concatenate([[1.0], c])


def horner_f32(c32: np.ndarray, f: np.ndarray) -> np.ndarray:
    """p(f) evaluated as the kernel does: Horner with one fp32 rounding per FMA."""
    f = np.asarray(f, dtype=np.float32)
    p = np.full_like(f, c32[-1], dtype=np.float32)
    for a in c32[-2::-1]:
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(a)).astype(np.float32)
    return p


def max_rel_error(c32: np.ndarray) -> float:
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    ref = np.exp2(f.astype(np.float64))
    return float(np.max(np.abs(horner_f32(c32, f).astype(np.float64) - ref) / ref))


def main():
    c32 = fit().astype(np.float32)
    print(f"// degree {DEGREE}, p(0) = 1, max relative error of fp32 Horner on [-1/2, 1/2]: "
          f"{max_rel_error(c32):.3e}")
    for i, a in enumerate(c32[1:], start=1):
        mant, ex = float(a).hex().split("p")
        print(f"constexpr float kExp2C{i} = {mant.rstrip('0')}p{ex}f;  // {float(a):.9g}")


if __name__ == "__main__":
    main()
