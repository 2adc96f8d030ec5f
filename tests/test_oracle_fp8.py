"""Pins for the E4M3 oracle (oracle/fp8.py): the decoder against closed-form codes and
against torch's float8_e4m3fn conversion of all 256 codes (a library routine), and the
attention against the float64 attention oracle on library-decoded inputs. Planted
mistakes in the decoder must fail a pin. CPU only."""
import os
import types

import numpy as np
import pytest
import torch

from oracle import attention_f64, attention_fp8_f64, attention_fp8_rows_f64, e4m3_to_f64
from workloads import make_fp8_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "fp8.py")

CLOSED_FORM = {0x00: 0.0, 0x38: 1.0, 0xB8: -1.0, 0x40: 2.0, 0xC0: -2.0, 0x7E: 448.0,
               0xFE: -448.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
               0x3C: 1.5, 0x30: 0.5, 0x77: 240.0}


def pin_closed_form(decode):
    for code, val in CLOSED_FORM.items():
        assert decode(np.array([code], dtype=np.uint8))[0] == val, hex(code)
    assert np.isnan(decode(np.array([0x7F, 0xFF], dtype=np.uint8))).all()
    assert np.signbit(decode(np.array([0x80], dtype=np.uint8))[0])


def pin_library_all_codes(decode):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float32).double().numpy()
    ours = decode(codes.numpy())
    nan = np.isnan(lib)
    assert np.array_equal(nan, np.isnan(ours))
    assert np.array_equal(lib[~nan], ours[~nan])


PINS = [pin_closed_form, pin_library_all_codes]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(e4m3_to_f64)


@pytest.mark.parametrize("causal", [False, True])
def test_attention_equals_definition_on_library_decoded_inputs(causal):
    q8, k8, v8, dq, dk, dv = make_fp8_inputs(1, 4, 2, 37, 53, 16, seed=3)
    lib = lambda c, s: c.view(torch.float8_e4m3fn).to(torch.float32).double().numpy() * s
    O, L = attention_fp8_f64(q8, k8, v8, dq, dk, dv, causal, 0.25)
    Oe, Le = attention_f64(lib(q8, dq), lib(k8, dk), lib(v8, dv), causal, 0.25)
    np.testing.assert_array_equal(O, Oe)
    np.testing.assert_array_equal(L, Le)
    rows = np.array([0, 5, 36])
    for h in range(4):
        Or, Lr = attention_fp8_rows_f64(q8, k8, v8, dq, dk, dv, causal, 0.25, 0, h, rows)
        np.testing.assert_allclose(Or, O[0, h, rows], rtol=0, atol=1e-15)
        np.testing.assert_allclose(Lr, L[0, h, rows], rtol=0, atol=1e-13)


def test_generator_uses_the_full_range():
    q8, k8, v8, dq, dk, dv = make_fp8_inputs(2, 2, 1, 64, 64, 32, seed=5)
    for c, s in ((q8, dq), (k8, dk), (v8, dv)):
        vals = e4m3_to_f64(c)
        assert np.isfinite(vals).all() and np.abs(vals).max() == 448.0 and s > 0


MUTANTS = {
    "exponent bias 8": ("np.exp2(exp - 7.0)", "np.exp2(exp - 8.0)"),
    "no implicit one": ("(1.0 + man / 8.0)", "(man / 8.0)"),
    "subnormals as normals": ("out = np.where(exp == 0, subnormal, normal)", "out = normal"),
    "sign dropped": ("sign = np.where(c & 0x80, -1.0, 1.0)", "sign = np.ones(c.shape)"),
    "mantissa over 16": ("(1.0 + man / 8.0)", "(1.0 + man / 16.0)"),
    "saturating instead of NaN": ("return np.where((exp == 15) & (man == 7), np.nan, out)", "return out"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    with open(SRC) as f:
        src = f.read()
    assert old in src, f"mutation anchor not found: {old!r}"
    mod = types.ModuleType("oracle.fp8_mutant")
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new, 1), "fp8_mutant", "exec"), mod.__dict__)
    failed = []
    for pin in PINS:
        try:
            pin(mod.e4m3_to_f64)
        except Exception as e:
            failed.append((pin.__name__, type(e).__name__))
    assert failed, f"mutant {name!r} passed every pin"


# ---- descale identities (hypothesis) -------------------------------------------------
from hypothesis import HealthCheck, given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402

SETTINGS = settings(derandomize=True, max_examples=40, deadline=None,
                    suppress_health_check=[HealthCheck.too_slow])


def _codes(rng, shape):
    """Random finite E4M3 codes (the two NaN codes excluded)."""
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    return np.where((c & 0x7F) == 0x7F, c & 0xF0, c).astype(np.uint8)


@SETTINGS
@given(st.integers(0, 2**31 - 1), st.booleans(), st.floats(2.0 ** -8, 2.0 ** -2),
       st.floats(2.0 ** -8, 2.0 ** -2), st.floats(1e-3, 10.0), st.floats(0.25, 4.0))
def test_descales_fold_as_the_definition_says(seed, causal, dq, dk, dv, alpha):
    """Q and K descales multiply the scores (so they fold into the scale), V's descale
    multiplies O and leaves the LSE alone."""
    rng = np.random.default_rng(seed)
    Hkv = int(rng.integers(1, 3))
    Hq = Hkv * int(rng.integers(1, 3))
    Nq, Nk = int(rng.integers(1, 12)), int(rng.integers(1, 12))
    q8, k8, v8 = _codes(rng, (1, Hq, Nq, 8)), _codes(rng, (1, Hkv, Nk, 8)), _codes(rng, (1, Hkv, Nk, 8))
    s = 0.3
    O, L = attention_fp8_f64(q8, k8, v8, dq, dk, dv, causal, s)
    O2, L2 = attention_fp8_f64(q8, k8, v8, dq * alpha, dk, dv, causal, s / alpha)
    O3, L3 = attention_fp8_f64(q8, k8, v8, dq, dk * alpha, dv, causal, s / alpha)
    O4, L4 = attention_fp8_f64(q8, k8, v8, dq, dk, dv * alpha, causal, s)
    fin = np.isfinite(L)
    for Ox, Lx in ((O2, L2), (O3, L3)):
        assert np.allclose(Ox, O, rtol=1e-9, atol=1e-9 * max(1.0, float(np.abs(O).max())))
        assert np.array_equal(np.isfinite(Lx), fin) and np.allclose(Lx[fin], L[fin], rtol=1e-9, atol=1e-9)
    assert np.allclose(O4, alpha * O, rtol=1e-12, atol=0)
    assert np.array_equal(np.isfinite(L4), fin) and np.allclose(L4[fin], L[fin], rtol=0, atol=0)
