"""Property tests that pin the float64 attention oracle to identities of the definition
O = softmax(scale * Q K^T + mask) V (page "Kotaemon FlashAttention", attention formula and
exactness paragraph), over random shapes drawn by hypothesis. Each property is one that a
plausible slip in the oracle would break: a wrong operand order breaks linearity in V or
row equivariance, a wrong head mapping breaks the grouped-query identity, a misplaced
scale breaks the scale-folding identity, a mis-aligned causal mask breaks the single-row
and truncation identities, and mixed-up batch indexing breaks batch independence. The
tiled restatement, with and without the kernels' lazy running maximum and exponent
offset, must equal the definition for any tile sizes."""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import (attention_f64, attention_rows_f64, decode_f64, split_kv_decode_f64,
                    tiled_attention_f64)

SETTINGS = settings(derandomize=True, max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
ATOL = 1e-11


@st.composite
def shapes(draw, max_n=24):
    Hkv = draw(st.integers(1, 3))
    return dict(B=draw(st.integers(1, 2)), Hkv=Hkv, Hq=Hkv * draw(st.integers(1, 3)),
                Nq=draw(st.integers(1, max_n)), Nk=draw(st.integers(1, max_n)),
                d=draw(st.sampled_from([1, 4, 8])), seed=draw(st.integers(0, 2**31 - 1)),
                scale=draw(st.floats(0.05, 2.0)))


def make(s):
    r = np.random.default_rng(s["seed"])
    q = r.standard_normal((s["B"], s["Hq"], s["Nq"], s["d"]))
    k = r.standard_normal((s["B"], s["Hkv"], s["Nk"], s["d"]))
    v = r.standard_normal((s["B"], s["Hkv"], s["Nk"], s["d"]))
    return q, k, v, r


def close(a, b):
    fa, fb = np.isfinite(a), np.isfinite(b)
    return np.array_equal(fa, fb) and np.allclose(a[fa], b[fb], rtol=0, atol=ATOL) and \
        np.array_equal(a[~fa], b[~fb])


@SETTINGS
@given(shapes(), st.booleans(), st.floats(-3, 3), st.floats(-3, 3))
def test_linear_in_v(s, causal, a, b):
    """O is linear in V (the weights depend on Q and K only); LSE does not depend on V."""
    q, k, v1, r = make(s)
    v2 = r.standard_normal(v1.shape)
    O1, L1 = attention_f64(q, k, v1, causal, s["scale"])
    O2, _ = attention_f64(q, k, v2, causal, s["scale"])
    O3, L3 = attention_f64(q, k, a * v1 + b * v2, causal, s["scale"])
    assert close(O3, a * O1 + b * O2)
    assert close(L3, L1)


@SETTINGS
@given(shapes())
def test_query_rows_are_equivariant_without_mask(s):
    """Without the mask each output row depends only on its own query row: permuting the
    query rows permutes O and LSE the same way."""
    q, k, v, r = make(s)
    perm = r.permutation(s["Nq"])
    O1, L1 = attention_f64(q, k, v, False, s["scale"])
    O2, L2 = attention_f64(q[:, :, perm], k, v, False, s["scale"])
    assert close(O2, O1[:, :, perm]) and close(L2, L1[:, :, perm])


@SETTINGS
@given(shapes(), st.booleans())
def test_grouped_query_equals_repeated_kv_heads(s, causal):
    """Query head h reads KV head h // (Hq / Hkv): the grouped call equals multi-head
    attention on K, V with each KV head repeated Hq / Hkv times."""
    q, k, v, _ = make(s)
    g = s["Hq"] // s["Hkv"]
    O1, L1 = attention_f64(q, k, v, causal, s["scale"])
    O2, L2 = attention_f64(q, np.repeat(k, g, axis=1), np.repeat(v, g, axis=1), causal, s["scale"])
    assert close(O1, O2) and close(L1, L2)


@SETTINGS
@given(shapes(), st.booleans(), st.floats(0.25, 4.0))
def test_scale_folds_into_queries(s, causal, alpha):
    """Only scale * q.k enters: scaling the queries by alpha and the scale by 1 / alpha
    changes nothing."""
    q, k, v, _ = make(s)
    O1, L1 = attention_f64(q, k, v, causal, s["scale"])
    O2, L2 = attention_f64(q * alpha, k, v, causal, s["scale"] / alpha)
    assert np.allclose(O1, O2, rtol=0, atol=1e-10)
    fin = np.isfinite(L1)
    assert np.array_equal(fin, np.isfinite(L2)) and np.allclose(L1[fin], L2[fin], rtol=0, atol=1e-10)


@SETTINGS
@given(shapes())
def test_single_causal_row_sees_every_key(s):
    """Bottom-right alignment: with one query row, the causal mask hides no key."""
    q, k, v, _ = make(s)
    q1 = q[:, :, :1]
    assert all(close(a, b) for a, b in zip(attention_f64(q1, k, v, True, s["scale"]),
                                           attention_f64(q1, k, v, False, s["scale"])))


@SETTINGS
@given(shapes())
def test_causal_rows_equal_attention_over_their_visible_prefix(s):
    """Row i of a causal call sees keys 0 .. i + Nk - Nq: it equals non-causal attention of
    that one row over exactly those keys (no keys: O = 0, LSE = -inf)."""
    q, k, v, _ = make(s)
    Nq, Nk = s["Nq"], s["Nk"]
    O, L = attention_f64(q, k, v, True, s["scale"])
    for i in range(Nq):
        n = min(Nk, max(0, i + Nk - Nq + 1))
        if n == 0:
            assert np.all(O[:, :, i] == 0) and np.all(L[:, :, i] == -np.inf)
            continue
        Oi, Li = attention_f64(q[:, :, i:i + 1], k[:, :, :n], v[:, :, :n], False, s["scale"])
        assert close(O[:, :, i:i + 1], Oi) and close(L[:, :, i:i + 1], Li)


@SETTINGS
@given(shapes(), st.booleans())
def test_batches_are_independent(s, causal):
    """Each sequence of the batch is its own problem."""
    q, k, v, _ = make(s)
    O, L = attention_f64(q, k, v, causal, s["scale"])
    for b in range(s["B"]):
        Ob, Lb = attention_f64(q[b:b + 1], k[b:b + 1], v[b:b + 1], causal, s["scale"])
        assert close(O[b:b + 1], Ob) and close(L[b:b + 1], Lb)


@SETTINGS
@given(shapes(max_n=40), st.booleans(), st.integers(1, 40), st.integers(1, 40))
def test_tiled_restatement_matches_for_any_tile_sizes(s, causal, Br, Bc):
    """The online-softmax restatement (running max and normaliser over key tiles of Bc
    keys, query tiles of Br rows) equals the plain definition for any tile sizes."""
    q, k, v, _ = make(s)
    O, L = attention_f64(q, k, v, causal, s["scale"])
    g = s["Hq"] // s["Hkv"]
    for b in range(s["B"]):
        for h in range(s["Hq"]):
            Ot, Lt = tiled_attention_f64(q[b, h], k[b, h // g], v[b, h // g], causal, s["scale"],
                                         Br, Bc)
            assert close(Ot, O[b, h]) and close(Lt, L[b, h])


@SETTINGS
@given(shapes(max_n=40), st.booleans(), st.integers(1, 40), st.integers(1, 40),
       st.floats(0.0, 16.0), st.floats(-4.0, 8.0))
def test_lazy_rescale_and_exponent_offset_are_exact(s, causal, Br, Bc, tau, offset):
    """A running maximum that moves only when a tile's maximum passes it by more than
    2^tau, and an exponent offset taken back out of the LSE, leave O and LSE unchanged."""
    q, k, v, _ = make(s)
    O, L = attention_f64(q, k, v, causal, s["scale"])
    g = s["Hq"] // s["Hkv"]
    for b in range(s["B"]):
        for h in range(s["Hq"]):
            Ot, Lt = tiled_attention_f64(q[b, h], k[b, h // g], v[b, h // g], causal, s["scale"],
                                         Br, Bc, tau=tau, offset=offset)
            assert close(Ot, O[b, h]) and close(Lt, L[b, h])


@SETTINGS
@given(st.integers(0, 40), st.sampled_from([1, 4, 8]), st.integers(0, 2**31 - 1),
       st.floats(0.05, 2.0), st.lists(st.integers(0, 40), max_size=8))
def test_split_kv_decode_merge_is_exact(n, d, seed, scale, cuts):
    """Decode over keys cut into chunks (empty ones included), each chunk's (O, LSE) merged
    by the LSE weights, equals decode over all keys at once."""
    r = np.random.default_rng(seed)
    q = r.standard_normal((1, 1, d))
    k = r.standard_normal((1, 1, max(n, 1), d))
    v = r.standard_normal((1, 1, max(n, 1), d))
    bounds = [0] + sorted(min(c, n) for c in cuts) + [n]
    O, L = split_kv_decode_f64(q[0, 0], k[0, 0, :n], v[0, 0, :n], bounds, scale)
    Od, Ld = decode_f64(q, k, v, [n], scale)
    assert close(O, Od[0, 0]) and close(np.array(L), Ld[0, 0])


@SETTINGS
@given(shapes(), st.booleans(), st.data())
def test_sampled_rows_equal_the_full_result(s, causal, data):
    """The sampled-rows form (used on the largest workloads) gives exactly the full
    result's rows, for any subset in any order, repeats included, under either mask."""
    q, k, v, _ = make(s)
    O, L = attention_f64(q, k, v, causal, s["scale"])
    rows = np.array(data.draw(st.lists(st.integers(0, s["Nq"] - 1), min_size=1, max_size=12)))
    b = data.draw(st.integers(0, s["B"] - 1))
    h = data.draw(st.integers(0, s["Hq"] - 1))
    Or, Lr = attention_rows_f64(q, k, v, causal, s["scale"], b, h, rows)
    assert close(Or, O[b, h, rows]) and close(Lr, L[b, h, rows])
