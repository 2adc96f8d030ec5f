"""Pins for the per-sequence-length oracles (`attention_varlen_f64`,
`attention_paged_varlen_f64`), on the CPU.

* pure-Python brute force (math.exp, explicit loops) per sequence, on tiny ragged batches
  with empty query sets, empty key sets, more queries than keys (causal rows that see
  nothing), grouped-query heads and both mask modes;
* data past a sequence's lengths (query rows, key and value rows) never changes a result,
  even NaN;
* with every length at its maximum the oracle equals the uniform one;
* the paged form equals the contiguous one on the same tokens, pages scattered and the
  unused pool rows NaN;
* planted mistakes (the global length in place of the sequence's, a mask aligned to the
  batch's end, the lengths ignored) are each caught.
"""
import math
import os
import types

import numpy as np
import pytest
import torch

from oracle import attention_f64, attention_paged_varlen_f64, attention_varlen_f64
from workloads import make_page_table, paginate

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (B, Hq, Hkv, Nq, Nk, d, q_lens, kv_lens)
CASES = [
    (4, 2, 1, 5, 7, 3, [5, 0, 3, 4], [7, 4, 0, 2]),     # empty queries, empty keys, nq > nk
    (3, 4, 2, 6, 6, 2, [1, 6, 2], [6, 1, 5]),
    (2, 3, 3, 4, 9, 4, [4, 4], [9, 3]),
]


def _rand(seed, B, Hq, Hkv, Nq, Nk, d):
    r = np.random.default_rng(seed)
    return (r.standard_normal((B, Hq, Nq, d)), r.standard_normal((B, Hkv, Nk, d)),
            r.standard_normal((B, Hkv, Nk, d)))


def brute_force_check(fn):
    for seed, (B, Hq, Hkv, Nq, Nk, d, ql, kl) in enumerate(CASES):
        for causal in (False, True):
            scale = 0.7 + 0.1 * seed
            q, k, v = _rand(200 + seed, B, Hq, Hkv, Nq, Nk, d)
            O, L = fn(q, k, v, np.array(ql), np.array(kl), causal, scale)
            g = Hq // Hkv
            for b in range(B):
                nq, nk = ql[b], kl[b]
                for h in range(Hq):
                    for i in range(Nq):
                        if i >= nq:
                            assert np.all(np.isnan(O[b, h, i])) and np.isnan(L[b, h, i])
                            continue
                        vis = [j for j in range(nk) if (not causal) or j <= i + nk - nq]
                        if not vis:
                            assert np.all(O[b, h, i] == 0) and L[b, h, i] == -math.inf
                            continue
                        s = {j: scale * sum(q[b, h, i, t] * k[b, h // g, j, t] for t in range(d))
                             for j in vis}
                        z = math.fsum(math.exp(s[j]) for j in vis)
                        for t in range(d):
                            ref = math.fsum(math.exp(s[j]) * v[b, h // g, j, t] for j in vis) / z
                            assert abs(O[b, h, i, t] - ref) <= 1e-12 * max(1.0, abs(ref))
                        assert abs(L[b, h, i] - math.log(z)) <= 1e-12 * max(1.0, abs(math.log(z)))


def test_brute_force():
    brute_force_check(attention_varlen_f64)


def test_data_past_the_lengths_is_never_read():
    B, Hq, Hkv, Nq, Nk, d, ql, kl = CASES[0]
    q, k, v = _rand(7, B, Hq, Hkv, Nq, Nk, d)
    O, L = attention_varlen_f64(q, k, v, np.array(ql), np.array(kl), True, 0.5)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    for b in range(B):
        q2[b, :, ql[b]:] = np.nan
        k2[b, :, kl[b]:] = np.nan
        v2[b, :, kl[b]:] = np.nan
    O2, L2 = attention_varlen_f64(q2, k2, v2, np.array(ql), np.array(kl), True, 0.5)
    assert np.array_equal(O, O2, equal_nan=True) and np.array_equal(L, L2, equal_nan=True)


@pytest.mark.parametrize("causal", [False, True])
def test_full_lengths_equal_the_uniform_oracle(causal):
    q, k, v = _rand(9, 2, 4, 2, 6, 9, 3)
    O, L = attention_varlen_f64(q, k, v, np.array([6, 6]), np.array([9, 9]), causal, 0.6)
    Ou, Lu = attention_f64(q, k, v, causal, 0.6)
    assert np.array_equal(O, Ou) and np.array_equal(L, Lu)


@pytest.mark.parametrize("ps", [16, 32])
def test_paged_equals_contiguous(ps):
    B, Hq, Hkv, Nq, d = 3, 4, 2, 40, 8
    ql, kl = [40, 17, 0], [70, 33, 16]
    r = np.random.default_rng(11)
    q = torch.from_numpy(r.standard_normal((B, Hq, Nq, d)))
    kc = torch.from_numpy(r.standard_normal((B, Hkv, 80, d)))
    vc = torch.from_numpy(r.standard_normal((B, Hkv, 80, d)))
    lens = torch.tensor(kl)
    table, P = make_page_table(lens, ps, (80 + ps - 1) // ps, seed=3)
    kp, vp = paginate(kc, table, lens, ps, P), paginate(vc, table, lens, ps, P)   # unused rows NaN
    for causal in (False, True):
        O, L = attention_paged_varlen_f64(q, kp, vp, table, np.array(ql), np.array(kl), ps, causal, 0.4)
        Oc, Lc = attention_varlen_f64(q, kc, vc, np.array(ql), np.array(kl), causal, 0.4)
        assert np.array_equal(O, Oc, equal_nan=True) and np.array_equal(L, Lc, equal_nan=True)


SRC = os.path.join(ROOT, "oracle", "attention.py")
MUTANTS = {
    "global key count": ("K = _f64(k[b, h // g])[:nk]", "K = _f64(k[b, h // g])"),
    "mask aligned to the batch's end": ("visible_mask(rows, nq, nk, causal)",
                                        "visible_mask(rows, Nq, k.shape[2], causal)"),
    "query count ignored": ("visible_mask(rows, nq, nk, causal)", "visible_mask(rows, nk, nk, causal)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    with open(SRC) as f:
        src = f.read()
    assert old in src
    mod = types.ModuleType("oracle_varlen_mutant")
    exec(compile(src.replace(old, new, 1), "oracle_varlen_mutant", "exec"), mod.__dict__)
    with pytest.raises(Exception):
        brute_force_check(mod.attention_varlen_f64)
