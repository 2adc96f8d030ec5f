"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that every one
of them is caught by at least one pin. This is what makes the pins worth trusting."""
import os
import types

import pytest

from tests import oracle_pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "attention.py")

MUTANTS = {
    "dropped scale": ("S = scale * (Q @ K.T)", "S = (Q @ K.T)"),
    "scale applied twice": ("S = scale * (Q @ K.T)", "S = scale * scale * (Q @ K.T)"),
    "K and V swapped": ("K = _f64(k[b, h // g])", "K = _f64(v[b, h // g])"),
    "max dropped from LSE": ("lse[has] = m[has] + np.log(l[has])", "lse[has] = np.log(l[has])"),
    "wrong sign in exponent": ("E = np.exp(S - m_safe[:, None])", "E = np.exp(m_safe[:, None] - S)"),
    "no normalisation": ("O[has] = (E[has] / l[has, None]) @ V", "O[has] = E[has] @ V"),
    "top-left causal alignment": ("(np.asarray(rows)[:, None] + (Nk - Nq))", "(np.asarray(rows)[:, None])"),
    "strict causal mask": ("return cols <= (", "return cols < ("),
    "wrong GQA mapping": ("K = _f64(k[b, h // g])", "K = _f64(k[b, h % Hkv])"),
    "V rows reversed": ("O[has] = (E[has] / l[has, None]) @ V", "O[has] = (E[has] / l[has, None]) @ V[::-1]"),
    "log2 instead of ln": ("lse[has] = m[has] + np.log(l[has])", "lse[has] = m[has] + np.log2(l[has])"),
    "exp2 instead of exp": ("E = np.exp(S - m_safe[:, None])", "E = np.exp2(S - m_safe[:, None])"),
    "empty rows get LSE 0": ("lse = np.full(S.shape[0], -np.inf, dtype=np.float64)",
                             "lse = np.zeros(S.shape[0], dtype=np.float64)"),
}


def _load_mutant(old, new):
    with open(SRC) as f:
        src = f.read()
    assert old in src, f"mutation anchor not found: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new, 1), "oracle_mutant", "exec"), mod.__dict__)
    return mod.attention_f64


@pytest.mark.filterwarnings("ignore::RuntimeWarning")   # a broken mutant may form NaN/inf
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    attn = _load_mutant(*MUTANTS[name])
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(attn)
        except Exception as e:  # AssertionError, or a crash from the broken arithmetic
            failed.append((pin.__name__, type(e).__name__))
    assert failed, f"mutant {name!r} passed every pin"
