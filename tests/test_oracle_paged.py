"""Pins for the paged-cache oracle (oracle/paged.py), independent of its gather: a
brute-force per-token softmax written with scalar loops, invariance under a permutation of
the pool's pages, poisoned unused rows, and agreement with the contiguous-cache oracle.
A planted mistake in the gather must fail at least one of them. CPU only."""
import math
import os
import types

import numpy as np
import pytest
import torch

from oracle import decode_f64, attention_rows_f64
from oracle.paged import attention_paged_rows_f64, decode_paged_f64
from workloads import make_page_table, paginate

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "paged.py")


def _tiny_case():
    """ps = 2, pool of 6 pages in scrambled order, two sequences of 3 and 5 tokens."""
    rng = np.random.default_rng(5)
    ps, Hkv, Hq, d = 2, 1, 2, 3
    kpool = rng.standard_normal((6, Hkv, ps, d))
    vpool = rng.standard_normal((6, Hkv, ps, d))
    table = np.array([[4, 1, -1], [2, 5, 0]])
    lens = np.array([3, 5])
    q = rng.standard_normal((2, Hq, d))
    return q, kpool, vpool, table, lens, ps


def _brute_decode(q, kpool, vpool, table, lens, ps, scale):
    """Scalar loops: token t of sequence b is row t % ps of page table[b][t // ps]."""
    B, Hq, d = q.shape
    Hkv = kpool.shape[1]
    O = np.zeros((B, Hq, d))
    L = np.full((B, Hq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            kh = h // (Hq // Hkv)
            s = []
            for t in range(int(lens[b])):
                page, row = int(table[b][t // ps]), t % ps
                s.append(scale * sum(q[b, h, i] * kpool[page, kh, row, i] for i in range(d)))
            if not s:
                continue
            w = [math.exp(x) for x in s]
            tot = sum(w)
            for t in range(len(s)):
                page, row = int(table[b][t // ps]), t % ps
                for i in range(d):
                    O[b, h, i] += w[t] / tot * vpool[page, kh, row, i]
            L[b, h] = math.log(tot)
    return O, L


def pin_brute_force(decode_paged):
    q, kp, vp, table, lens, ps = _tiny_case()
    O, L = decode_paged(q, kp, vp, table, lens, ps, 0.8)
    Ob, Lb = _brute_decode(q, kp, vp, table, lens, ps, 0.8)
    np.testing.assert_allclose(O, Ob, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(L, Lb, rtol=1e-12, atol=1e-12)


def pin_page_permutation(decode_paged):
    """Relabelling the pool's pages (and the table with them) changes nothing."""
    q, kp, vp, table, lens, ps = _tiny_case()
    O, L = decode_paged(q, kp, vp, table, lens, ps, 0.8)
    perm = np.array([3, 0, 5, 1, 4, 2])                    # page p moves to perm[p]
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm], vp2[perm] = kp, vp
    table2 = np.where(table >= 0, perm[np.maximum(table, 0)], -1)
    O2, L2 = decode_paged(q, kp2, vp2, table2, lens, ps, 0.8)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(L, L2)


def pin_poisoned_unused_rows(decode_paged):
    """Pool rows no token maps to (row 1 of page 1, page 3, row 1 of page 0) may hold NaN."""
    q, kp, vp, table, lens, ps = _tiny_case()
    O, L = decode_paged(q, kp, vp, table, lens, ps, 0.8)
    kp2, vp2 = kp.copy(), vp.copy()
    for page, row in ((1, 1), (3, 0), (3, 1), (0, 1)):
        kp2[page, :, row] = np.nan
        vp2[page, :, row] = np.nan
    O2, L2 = decode_paged(q, kp2, vp2, table, lens, ps, 0.8)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(L, L2)


def pin_contiguous_cache(decode_paged):
    """A seeded paginated cache gives the contiguous-cache oracle's result."""
    rng = np.random.default_rng(9)
    B, Hq, Hkv, C, d, ps = 3, 4, 2, 40, 8, 8
    lens = np.array([40, 17, 1])
    kc = rng.standard_normal((B, Hkv, C, d))
    vc = rng.standard_normal((B, Hkv, C, d))
    q = rng.standard_normal((B, Hq, d))
    table, P = make_page_table(torch.tensor(lens), ps, 5, seed=2)
    kp = paginate(torch.from_numpy(kc), table, lens, ps, P).numpy()
    vp = paginate(torch.from_numpy(vc), table, lens, ps, P).numpy()
    O, L = decode_paged(q, kp, vp, table.numpy(), lens, ps, 0.3)
    Oc, Lc = decode_f64(q, kc, vc, lens, 0.3)
    np.testing.assert_allclose(O, Oc, rtol=0, atol=1e-14)
    np.testing.assert_allclose(L, Lc, rtol=0, atol=1e-14)


PINS = [pin_brute_force, pin_page_permutation, pin_poisoned_unused_rows, pin_contiguous_cache]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(decode_paged_f64)


def test_prefill_rows_match_contiguous():
    """attention_paged_rows_f64 equals the contiguous oracle on the gathered cache,
    bottom-right causal with a query chunk shorter than the keys."""
    rng = np.random.default_rng(3)
    Hq, Hkv, Nq, Nk, d, ps = 4, 2, 5, 21, 8, 4
    q = rng.standard_normal((1, Hq, Nq, d))
    kc = rng.standard_normal((1, Hkv, Nk, d))
    vc = rng.standard_normal((1, Hkv, Nk, d))
    table, P = make_page_table(torch.tensor([Nk]), ps, 7, seed=4)
    kp = paginate(torch.from_numpy(kc), table, [Nk], ps, P).numpy()
    vp = paginate(torch.from_numpy(vc), table, [Nk], ps, P).numpy()
    rows = np.arange(Nq)
    for causal in (False, True):
        for h in range(Hq):
            O, L = attention_paged_rows_f64(q, kp, vp, table.numpy(), Nk, ps, causal, 0.5, 0, h, rows)
            Oc, Lc = attention_rows_f64(q, kc, vc, causal, 0.5, 0, h, rows)
            np.testing.assert_allclose(O, Oc, rtol=0, atol=1e-14)
            np.testing.assert_allclose(L, Lc, rtol=0, atol=1e-14)


def test_page_table_generator():
    """Pages of different sequences are distinct, unused entries hold the fill value."""
    lens = torch.tensor([33, 0, 16, 1])
    table, P = make_page_table(lens, 16, 4, spare_pages=2, seed=1)
    assert P == 3 + 0 + 1 + 1 + 2
    used = [int(x) for x in table.flatten().tolist() if x >= 0]
    assert len(used) == len(set(used)) == P - 2
    assert table[1].tolist() == [-1] * 4 and table[0, 3].item() == -1


MUTANTS = {
    "page index off by one": ("out[:, t0:t1] = pool[int(table_row[j]), :, : t1 - t0]",
                              "out[:, t0:t1] = pool[int(table_row[min(j + 1, len(table_row) - 1)]), :, : t1 - t0]"),
    "rows taken from the page end": ("pool[int(table_row[j]), :, : t1 - t0]",
                                     "pool[int(table_row[j]), :, page_size - (t1 - t0):]"),
    "last partial page dropped": ("n_pages = (n_tokens + page_size - 1) // page_size",
                                  "n_pages = n_tokens // page_size"),
    "table row of the wrong sequence": ("K = gather_pages(kpool, table[b], n, page_size)[None]",
                                        "K = gather_pages(kpool, table[B - 1 - b], n, page_size)[None]"),
    "V gathered from K": ("V = gather_pages(vpool, table[b], n, page_size)[None]",
                          "V = gather_pages(kpool, table[b], n, page_size)[None]"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    with open(SRC) as f:
        src = f.read()
    assert old in src, f"mutation anchor not found: {old!r}"
    mod = types.ModuleType("oracle.paged_mutant")
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new, 1), "paged_mutant", "exec"), mod.__dict__)
    failed = []
    for pin in PINS:
        try:
            pin(mod.decode_paged_f64)
        except Exception as e:
            failed.append((pin.__name__, type(e).__name__))
    assert failed, f"mutant {name!r} passed every pin"
