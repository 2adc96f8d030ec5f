"""Property tests for the paged-cache and per-sequence-length oracles (`decode_paged_f64`,
`attention_paged_varlen_f64`, `attention_varlen_f64`), over random page sizes, lengths,
head groupings and page placements drawn by hypothesis. CPU only.

The pages are laid out here token by token (token t of sequence b is row t % page_size of
page table[b][t // page_size]), with a scalar loop of this file's own, so that neither the
oracle's gather nor the workload generator's slice copy is taken on trust. Every pool row
that no token maps to holds NaN: a gather that reads one shows it.

* the paged decode and the paged ragged-length oracle equal their contiguous forms on the
  same tokens, for any page size;
* relabelling the pool's pages (and the table with them) changes nothing;
* each sequence of a ragged batch equals the uniform oracle on that sequence's own query
  and key rows, its causal mask aligned to its own end; rows past its query length are NaN;
* data past a sequence's lengths is never read (NaN there changes nothing);
* single-token decode equals the ragged-length oracle with one query row per sequence;
* causal row i of a sequence with nq queries and nk keys equals decode of that one query
  over the first i + nk - nq + 1 keys (a different code path: truncation, not a mask).
"""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import (attention_f64, attention_paged_varlen_f64, attention_varlen_f64,
                    decode_f64, decode_paged_f64)

SETTINGS = settings(derandomize=True, max_examples=60, deadline=None,
                    suppress_health_check=[HealthCheck.too_slow])
ATOL = 1e-12


@st.composite
def ragged(draw, max_n=20):
    Hkv = draw(st.integers(1, 3))
    B = draw(st.integers(1, 4))
    Nq = draw(st.integers(1, max_n))
    Nk = draw(st.integers(1, max_n))
    return dict(B=B, Hkv=Hkv, Hq=Hkv * draw(st.integers(1, 3)), Nq=Nq, Nk=Nk,
                d=draw(st.sampled_from([1, 3, 8])),
                q_lens=draw(st.lists(st.integers(0, Nq), min_size=B, max_size=B)),
                kv_lens=draw(st.lists(st.integers(0, Nk), min_size=B, max_size=B)),
                page_size=draw(st.integers(1, 8)), spare=draw(st.integers(0, 4)),
                seed=draw(st.integers(0, 2**31 - 1)), scale=draw(st.floats(0.05, 2.0)))


def make(s):
    r = np.random.default_rng(s["seed"])
    q = r.standard_normal((s["B"], s["Hq"], s["Nq"], s["d"]))
    k = r.standard_normal((s["B"], s["Hkv"], s["Nk"], s["d"]))
    v = r.standard_normal((s["B"], s["Hkv"], s["Nk"], s["d"]))
    return q, k, v, r


def scatter(k, v, lens, ps, spare, r):
    """Pools [P, Hkv, ps, d] (NaN where no token lands) and a table [B, max_pages]: every
    sequence's pages are drawn from one random permutation of the pool, entries past a
    sequence's last page are -1."""
    B, Hkv, Nk, d = k.shape
    need = [-(-int(n) // ps) for n in lens]
    P = sum(need) + spare
    perm = r.permutation(P)
    table = np.full((B, max(1, -(-Nk // ps))), -1, dtype=np.int64)
    at = 0
    for b in range(B):
        table[b, :need[b]] = perm[at:at + need[b]]
        at += need[b]
    kpool = np.full((P, Hkv, ps, d), np.nan)
    vpool = np.full((P, Hkv, ps, d), np.nan)
    for b in range(B):
        for t in range(int(lens[b])):
            page, row = table[b, t // ps], t % ps
            kpool[page, :, row] = k[b, :, t]
            vpool[page, :, row] = v[b, :, t]
    return kpool, vpool, table


def close(a, b, atol=ATOL):
    """Equal within atol where finite; NaN and +-inf in exactly the same places."""
    fa, fb = np.isfinite(a), np.isfinite(b)
    return np.array_equal(fa, fb) and np.allclose(a[fa], b[fb], rtol=0, atol=atol) and \
        np.array_equal(np.isnan(a), np.isnan(b)) and \
        np.array_equal(a[np.isinf(a)], b[np.isinf(b)])


@SETTINGS
@given(ragged())
def test_paged_decode_equals_contiguous(s):
    q, k, v, r = make(s)
    q1 = q[:, :, 0]
    kpool, vpool, table = scatter(k, v, s["kv_lens"], s["page_size"], s["spare"], r)
    Op, Lp = decode_paged_f64(q1, kpool, vpool, table, s["kv_lens"], s["page_size"], s["scale"])
    Oc, Lc = decode_f64(q1, k, v, s["kv_lens"], s["scale"])
    assert close(Op, Oc) and close(Lp, Lc)


@SETTINGS
@given(ragged(), st.booleans())
def test_paged_varlen_equals_contiguous(s, causal):
    q, k, v, r = make(s)
    kpool, vpool, table = scatter(k, v, s["kv_lens"], s["page_size"], s["spare"], r)
    Op, Lp = attention_paged_varlen_f64(q, kpool, vpool, table, s["q_lens"], s["kv_lens"],
                                        s["page_size"], causal, s["scale"])
    Oc, Lc = attention_varlen_f64(q, k, v, s["q_lens"], s["kv_lens"], causal, s["scale"])
    assert close(Op, Oc) and close(Lp, Lc)


@SETTINGS
@given(ragged(), st.booleans())
def test_relabelling_pool_pages_changes_nothing(s, causal):
    q, k, v, r = make(s)
    kpool, vpool, table = scatter(k, v, s["kv_lens"], s["page_size"], s["spare"], r)
    pi = r.permutation(kpool.shape[0])                 # page p moves to slot pi[p]
    kpool2, vpool2 = np.empty_like(kpool), np.empty_like(vpool)
    kpool2[pi], vpool2[pi] = kpool, vpool
    table2 = np.array([[pi[t] if t >= 0 else -1 for t in row] for row in table], dtype=np.int64)
    args = (s["q_lens"], s["kv_lens"], s["page_size"], causal, s["scale"])
    O1, L1 = attention_paged_varlen_f64(q, kpool, vpool, table, *args)
    O2, L2 = attention_paged_varlen_f64(q, kpool2, vpool2, table2, *args)
    assert close(O1, O2, atol=0) and close(L1, L2, atol=0)


@SETTINGS
@given(ragged(), st.booleans())
def test_each_sequence_is_its_own_uniform_problem(s, causal):
    q, k, v, _ = make(s)
    O, L = attention_varlen_f64(q, k, v, s["q_lens"], s["kv_lens"], causal, s["scale"])
    for b in range(s["B"]):
        nq, nk = s["q_lens"][b], s["kv_lens"][b]
        assert np.all(np.isnan(O[b, :, nq:])) and np.all(np.isnan(L[b, :, nq:]))
        if nq == 0:
            continue
        if nk == 0:                                   # no keys: O = 0, LSE = -inf
            assert np.all(O[b, :, :nq] == 0) and np.all(L[b, :, :nq] == -np.inf)
            continue
        Ou, Lu = attention_f64(q[b:b + 1, :, :nq], k[b:b + 1, :, :nk], v[b:b + 1, :, :nk],
                               causal, s["scale"])
        assert close(O[b:b + 1, :, :nq], Ou) and close(L[b:b + 1, :, :nq], Lu)


@SETTINGS
@given(ragged(), st.booleans())
def test_data_past_the_lengths_is_never_read(s, causal):
    q, k, v, _ = make(s)
    O1, L1 = attention_varlen_f64(q, k, v, s["q_lens"], s["kv_lens"], causal, s["scale"])
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    for b in range(s["B"]):
        q2[b, :, s["q_lens"][b]:] = np.nan
        k2[b, :, s["kv_lens"][b]:] = np.nan
        v2[b, :, s["kv_lens"][b]:] = np.nan
    O2, L2 = attention_varlen_f64(q2, k2, v2, s["q_lens"], s["kv_lens"], causal, s["scale"])
    assert close(O1, O2, atol=0) and close(L1, L2, atol=0)


@SETTINGS
@given(ragged(), st.booleans())
def test_decode_is_one_query_row_per_sequence(s, causal):
    """One query row sees every key under either mask (bottom-right alignment)."""
    q, k, v, _ = make(s)
    q1 = q[:, :, :1]
    Od, Ld = decode_f64(q1[:, :, 0], k, v, s["kv_lens"], s["scale"])
    Ov, Lv = attention_varlen_f64(q1, k, v, [1] * s["B"], s["kv_lens"], causal, s["scale"])
    assert close(Ov[:, :, 0], Od) and close(Lv[:, :, 0], Ld)


@SETTINGS
@given(ragged())
def test_causal_row_is_decode_over_its_visible_prefix(s):
    q, k, v, _ = make(s)
    O, L = attention_varlen_f64(q, k, v, s["q_lens"], s["kv_lens"], True, s["scale"])
    for b in range(s["B"]):
        nq, nk = s["q_lens"][b], s["kv_lens"][b]
        for i in range(nq):
            n = [max(0, min(nk, i + nk - nq + 1))]
            Od, Ld = decode_f64(q[b:b + 1, :, i], k[b:b + 1], v[b:b + 1], n, s["scale"])
            assert close(O[b, :, i], Od[0]) and close(L[b, :, i], Ld[0])
