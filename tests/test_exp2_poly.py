"""CPU checks of exp2_emu, the FMA-pipe 2^x that the softmax uses for 2 of every 16
exponential pairs with 64-key tiles (d = 64).

The device code evaluates 2^x as 2^j * p(f): x clamped to >= -127, j = round-to-nearest(x)
through the 1.5 * 2^23 shifter, f = x - j, p(f) = 1 + f (c1 + f (c2 + f (c3 + f c4))) fitted
by io_aware_exact_28_b200/csrc/fit_exp2_poly.py, and j added to the exponent field as an
integer. These tests check that the constants compiled into sm100.cuh are the fit's, that
the fit meets its error bound, and that the reduction + polynomial + exponent arithmetic,
replayed step for step in fp32 with NumPy, stays within that bound of the true 2^x over
the range the softmax uses and gives exactly +0 for masked keys (x = -inf). The GPU
parity tests cover the compiled code.
"""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "io_aware_exact_28_b200", "csrc")
sys.path.insert(0, CSRC)
import fit_exp2_poly  # noqa: E402

SHIFTER = np.float32(12582912.0)   # 1.5 * 2^23


def header_coefficients():
    with open(os.path.join(CSRC, "sm100.cuh")) as f:
        src = f.read()
    found = dict(re.findall(r"constexpr float kExp2C(\d) = (0x[0-9a-fA-Fp.+-]+)f;", src))
    assert sorted(found) == ["1", "2", "3", "4"], found
    return np.array([1.0] + [float.fromhex(found[str(i)]) for i in range(1, 5)], dtype=np.float32)


def emu(x):
    """The device function's steps in fp32 (integer steps mod 2^32)."""
    x = np.asarray(x, dtype=np.float32)
    with np.errstate(invalid="ignore"):
        xc = np.fmax(x, np.float32(-127.0))
    t = (xc + SHIFTER).astype(np.float32)
    f = (xc - (t - SHIFTER).astype(np.float32)).astype(np.float32)
    p = fit_exp2_poly.horner_f32(header_coefficients(), f)
    bits = (p.view(np.uint32).astype(np.uint64) +
            (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) & np.uint64(0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32), f


def test_header_constants_match_the_fit():
    fitted = fit_exp2_poly.fit().astype(np.float32)
    assert fitted[0] == 1.0
    assert np.array_equal(header_coefficients(), fitted)


def test_polynomial_error_bound():
    assert fit_exp2_poly.max_rel_error(header_coefficients()) < 3e-6


def test_fit_reduces_to_taylor_terms():
    # Near f = 0 the fit must agree with the Taylor series of 2^f = e^(f ln 2): the linear
    # coefficient is ln 2 and the quadratic (ln 2)^2 / 2, to the accuracy of a minimax fit.
    c = fit_exp2_poly.fit()
    assert abs(c[1] - np.log(2.0)) < 1e-4
    assert abs(c[2] - np.log(2.0) ** 2 / 2) < 1e-3


def test_reduction_and_scaling_replayed_in_fp32():
    x = np.concatenate([np.linspace(-126.0, 12.0, 400001), [-0.5, 0.5, 0.0, 7.999, -1e-7, 12.0]])
    r, f = emu(x)
    assert np.all(np.abs(f) <= 0.5)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(r.astype(np.float64) - ref) / ref
    assert rel.max() < 4e-6, rel.max()
    # integer powers of two are exact
    k = np.arange(-126, 13, dtype=np.float32)
    assert np.array_equal(emu(k)[0], np.exp2(k))


def test_masked_and_underflowing_inputs():
    # -inf (masked key), the clamp itself and anything below it give +0 exactly.
    r, _ = emu(np.array([-np.inf, -127.0, -127.5, -200.0, -1e30], dtype=np.float32))
    assert np.all(r.view(np.uint32) == 0)
    # between the clamp and the smallest normal: tiny, positive, never garbage
    x = np.linspace(-126.99, -126.0, 1001).astype(np.float32)
    r, _ = emu(x)
    assert np.all(r >= 0) and np.all(r <= np.float32(2.0 ** -125))
    assert np.all(np.isfinite(r))
