"""CPU checks of the FMA-pipe exp2 used in the prefill softmax.

The device code evaluates 2^x as 2^j * p(f) with j = round(x), f = x - j, and a degree-4
polynomial p fitted by io_aware_exact_28_b200/csrc/fit_exp2_poly.py. These tests check
that the constants compiled into sm100.cuh are exactly what the fitting script produces,
and that the reduction + polynomial + exponent-field scaling, replayed step for step in
fp32 with NumPy, stays within its stated error bound of the true 2^x over the range the
kernel uses. The GPU parity tests (LSE to 1e-4) cover the compiled code itself.
"""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "io_aware_exact_28_b200", "csrc")
sys.path.insert(0, CSRC)
import fit_exp2_poly  # noqa: E402


def header_coefficients():
    with open(os.path.join(CSRC, "sm100.cuh")) as f:
        src = f.read()
    found = dict(re.findall(r"constexpr float kExp2C(\d) = (0x[0-9a-fA-Fp.+-]+)f;", src))
    return np.array([float.fromhex(found[str(i)]) for i in range(len(found))], dtype=np.float32)


def test_header_constants_match_the_fit():
    fitted = fit_exp2_poly.fit().astype(np.float32)
    assert np.array_equal(header_coefficients(), fitted)


def test_polynomial_error_bound():
    assert fit_exp2_poly.max_rel_error(header_coefficients()) < 3e-6


def test_reduction_and_scaling_replayed_in_fp32():
    c = header_coefficients()
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), [-0.5, 0.5, 0.0, 7.999, -1e-7]]).astype(np.float32)
    xc = np.maximum(x, np.float32(-126.0))
    shifter = np.float32(12582912.0)
    t = (xc + shifter).astype(np.float32)
    f = (xc - (t - shifter)).astype(np.float32)
    assert np.all(np.abs(f) <= 0.5)
    p = fit_exp2_poly.horner_f32(c, f)
    j_bits = (t.view(np.uint32).astype(np.uint64) << np.uint64(23)) & np.uint64(0xFFFFFFFF)
    r = ((p.view(np.uint32).astype(np.uint64) + j_bits) & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(r.astype(np.float64) - ref) / ref
    assert rel.max() < 4e-6, rel.max()
    # below the clamp the result is a tiny positive number, never garbage or negative
    y = np.float32(-126.0)
    t = np.float32(y + shifter)
    assert ((int(t.view(np.uint32)) << 23) & 0xFFFFFFFF) == ((-126 << 23) & 0xFFFFFFFF)
