"""Pins for the float64 oracle: properties fixed by the pages and by mathematics.

Each pin takes the attention function under test (signature of
``oracle.attention_f64``: ``(q, k, v, causal, scale) -> (O, LSE)``) and raises
AssertionError when it is violated. `test_oracle_pins.py` runs them on the oracle;
`test_oracle_mutants.py` runs them on deliberately broken copies of the oracle to
show that each plausible mistake is caught by at least one pin.

None of these re-types the oracle's own code path: they use closed forms, pure-Python
brute force with `math.exp`, a library routine (torch's float64 CPU
scaled_dot_product_attention, the call the pages make), hand-worked fixtures, and
invariances of the definition.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_worked.json")


def _rng(seed):
    return np.random.default_rng(seed)


def _rand(seed, B, Hq, Hkv, Nq, Nk, d):
    r = _rng(seed)
    return (r.standard_normal((B, Hq, Nq, d)), r.standard_normal((B, Hkv, Nk, d)),
            r.standard_normal((B, Hkv, Nk, d)))


def _n_visible(i, Nq, Nk, causal):
    return Nk if not causal else max(0, min(Nk, i + (Nk - Nq) + 1))


# ---------------------------------------------------------------------------------------
def pin_golden(attn):
    """Hand-worked examples with exact answers (tests/golden/hand_worked.json)."""
    def ev(s):
        s = s.strip()
        if s == "-inf":
            return -math.inf
        if s.startswith("2*ln("):
            return 2 * math.log(float(Fraction(s[5:-1])))
        if s.startswith("ln("):
            return math.log(float(Fraction(s[3:-1])))
        return float(Fraction(s))

    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q = np.array([[[ev(x) for x in row] for row in h] for h in c["q"]])[None]
        k = np.array([[[ev(x) for x in row] for row in h] for h in c["k"]])[None]
        v = np.array([[[ev(x) for x in row] for row in h] for h in c["v"]])[None]
        o = np.array([[[ev(x) for x in row] for row in h] for h in c["o"]])[None]
        lse = np.array([[ev(x) for x in h] for h in c["lse"]])[None]
        O, L = attn(q, k, v, c["causal"], ev(c["scale"]))
        assert np.allclose(O, o, rtol=0, atol=1e-12), (c["name"], O, o)
        fin = np.isfinite(lse)
        assert np.array_equal(np.isfinite(L), fin), (c["name"], L, lse)
        assert np.allclose(L[fin], lse[fin], rtol=0, atol=1e-12), (c["name"], L, lse)


def pin_brute_force(attn):
    """Element-by-element pure-Python attention (math.exp, explicit loops) on tiny inputs,
    over square and rectangular causal masks, GQA and non-unit scales."""
    cases = [(1, 1, 1, 5, 5, 3, True, 0.7), (1, 2, 2, 4, 6, 2, True, 0.5),
             (2, 4, 2, 3, 3, 4, False, 0.5), (1, 2, 1, 6, 4, 3, True, 1.3),
             (1, 3, 3, 1, 7, 2, False, 0.9)]
    for seed, (B, Hq, Hkv, Nq, Nk, d, causal, scale) in enumerate(cases):
        q, k, v = _rand(100 + seed, B, Hq, Hkv, Nq, Nk, d)
        O, L = attn(q, k, v, causal, scale)
        g = Hq // Hkv
        for b in range(B):
            for h in range(Hq):
                kh = h // g
                for i in range(Nq):
                    vis = [j for j in range(Nk) if (not causal) or j <= i + Nk - Nq]
                    if not vis:
                        assert all(O[b, h, i, t] == 0 for t in range(d))
                        assert L[b, h, i] == -math.inf
                        continue
                    s = {j: scale * sum(q[b, h, i, t] * k[b, kh, j, t] for t in range(d))
                         for j in vis}
                    z = math.fsum(math.exp(s[j]) for j in vis)
                    for t in range(d):
                        ref = math.fsum(math.exp(s[j]) * v[b, kh, j, t] for j in vis) / z
                        assert abs(O[b, h, i, t] - ref) <= 1e-12 * max(1.0, abs(ref)), \
                            (b, h, i, t, O[b, h, i, t], ref)
                    assert abs(L[b, h, i] - math.log(z)) <= 1e-12 * max(1.0, abs(math.log(z)))


def pin_library_sdpa(attn):
    """torch float64 CPU scaled_dot_product_attention (the routine the pages call) as an
    independent special case: square causal and non-causal, rectangular with an explicit
    bottom-right boolean mask, and grouped-query heads."""
    import torch
    import torch.nn.functional as F
    cases = [(2, 3, 3, 33, 33, 16, True), (1, 4, 2, 20, 45, 8, True),
             (1, 4, 1, 17, 17, 8, False), (2, 2, 2, 9, 30, 32, False)]
    for seed, (B, Hq, Hkv, Nq, Nk, d, causal) in enumerate(cases):
        q, k, v = _rand(200 + seed, B, Hq, Hkv, Nq, Nk, d)
        scale = 1.0 / math.sqrt(d)
        O, L = attn(q, k, v, causal, scale)
        tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
        mask = None
        if causal:
            i = torch.arange(Nq)[:, None]
            j = torch.arange(Nk)[None, :]
            mask = j <= i + (Nk - Nq)
        ref = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=scale,
                                             enable_gqa=(Hq != Hkv)).numpy()
        assert np.allclose(O, ref, rtol=0, atol=1e-12), np.abs(O - ref).max()
        kk = np.repeat(k, Hq // Hkv, axis=1)
        s = scale * np.einsum("bhid,bhjd->bhij", q, kk)
        if causal:
            s = np.where(mask.numpy(), s, -np.inf)
        ref_lse = torch.logsumexp(torch.from_numpy(s), dim=-1).numpy()
        assert np.allclose(L, ref_lse, rtol=0, atol=1e-12)


def pin_row_sums(attn):
    """Rows of P = exp(S - LSE) sum to 1 (|sum - 1| <= 1e-12), scores summed with
    math.fsum from explicit dot products."""
    for seed, (Nq, Nk, causal) in enumerate([(7, 7, True), (5, 9, True), (6, 4, False)]):
        q, k, v = _rand(300 + seed, 1, 2, 2, Nq, Nk, 5)
        scale = 0.6
        _, L = attn(q, k, v, causal, scale)
        for h in range(2):
            for i in range(Nq):
                vis = [j for j in range(Nk) if (not causal) or j <= i + Nk - Nq]
                tot = math.fsum(math.exp(scale * math.fsum(q[0, h, i] * k[0, h, j]) - L[0, h, i])
                                for j in vis)
                assert abs(tot - 1.0) <= 1e-12, (h, i, tot)


def pin_constant_v(attn):
    """Every V row equal to the same vector c gives O = c on every row with a visible key."""
    q, k, _ = _rand(400, 2, 4, 2, 40, 40, 8)
    c = _rng(401).standard_normal(8)
    v = np.broadcast_to(c, (2, 2, 40, 8)).copy()
    for causal in (False, True):
        O, _ = attn(q, k, v, causal, 0.35)
        assert np.allclose(O, np.broadcast_to(c, O.shape), rtol=0, atol=1e-12)


def pin_causal_first_row(attn):
    """Square causal: row 0 sees only key 0, so O[0] = V[0] and LSE[0] = scale*q0.k0."""
    q, k, v = _rand(500, 2, 2, 2, 31, 31, 16)
    O, L = attn(q, k, v, True, 0.25)
    assert np.allclose(O[:, :, 0], v[:, :, 0], rtol=0, atol=1e-12)
    s00 = 0.25 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0])
    assert np.allclose(L[:, :, 0], s00, rtol=0, atol=1e-12)


def pin_zero_query(attn):
    """Q = 0: every visible score is 0, so O_i = mean of the visible V rows and
    LSE_i = ln(#visible); rows with no visible key give O = 0, LSE = -inf."""
    for (Nq, Nk, causal) in [(12, 12, True), (5, 11, True), (9, 4, True), (6, 10, False)]:
        _, k, v = _rand(600 + Nq, 1, 2, 1, Nq, Nk, 3)
        q = np.zeros((1, 2, Nq, 3))
        O, L = attn(q, k, v, causal, 0.8)
        for h in range(2):
            for i in range(Nq):
                n = _n_visible(i, Nq, Nk, causal)
                if n == 0:
                    assert np.all(O[0, h, i] == 0) and L[0, h, i] == -np.inf
                    continue
                assert np.allclose(O[0, h, i], v[0, 0, :n].mean(axis=0), rtol=0, atol=1e-12)
                assert abs(L[0, h, i] - math.log(n)) <= 1e-12


def pin_one_hot(attn):
    """Q row = c*e1 and K row j* = e1 with all other K rows 0, c*scale = 400: the weight
    of every other key is exp(-400) (zero in float64 next to 1), so O = V[j*]."""
    Nk, d = 24, 8
    k = np.zeros((1, 1, Nk, d))
    jstar = 17
    k[0, 0, jstar, 0] = 1.0
    v = _rng(700).standard_normal((1, 1, Nk, d))
    q = np.zeros((1, 1, 3, d))
    q[0, 0, :, 0] = 800.0
    O, L = attn(q, k, v, False, 0.5)
    assert np.allclose(O[0, 0], np.broadcast_to(v[0, 0, jstar], (3, d)), rtol=0, atol=1e-12)
    assert np.allclose(L[0, 0], 400.0, rtol=0, atol=1e-9)


def pin_key_permutation(attn):
    """Non-causal attention is invariant to a joint permutation of the K and V rows."""
    q, k, v = _rand(800, 1, 3, 3, 10, 26, 8)
    perm = _rng(801).permutation(26)
    O1, L1 = attn(q, k, v, False, 0.4)
    O2, L2 = attn(q, k[:, :, perm], v[:, :, perm], False, 0.4)
    assert np.allclose(O1, O2, rtol=0, atol=1e-12) and np.allclose(L1, L2, rtol=0, atol=1e-12)


def pin_key_shift(attn):
    """Adding a vector c to every key adds scale*q_i.c to every score of row i: O is
    unchanged and LSE_i moves by exactly scale*q_i.c."""
    q, k, v = _rand(900, 1, 2, 2, 14, 14, 6)
    c = _rng(901).standard_normal(6)
    for causal in (False, True):
        O1, L1 = attn(q, k, v, causal, 0.5)
        O2, L2 = attn(q, k + c, v, causal, 0.5)
        assert np.allclose(O1, O2, rtol=0, atol=1e-11)
        assert np.allclose(L2 - L1, 0.5 * np.einsum("bhid,d->bhi", q, c), rtol=0, atol=1e-11)


ALL_PINS = [pin_golden, pin_brute_force, pin_library_sdpa, pin_row_sums, pin_constant_v,
            pin_causal_first_row, pin_zero_query, pin_one_hot, pin_key_permutation,
            pin_key_shift]
