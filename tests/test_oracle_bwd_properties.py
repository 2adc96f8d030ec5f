"""Property tests that pin the float64 backward oracle (gradients of
O = softmax(scale * Q K^T + mask) V) to identities of that definition, over random shapes
drawn by hypothesis:

* every row of dS = P * (dP - D) sums to zero, because D_i = sum_j P_ij dP_ij and the
  row of P sums to one; adding one vector to every key therefore leaves dQ, dK and dV
  unchanged (the forward's P does not move either);
* the gradients are linear in the upstream gradient dO;
* only scale * q.k enters: scaling Q by alpha and the scale by 1 / alpha divides dQ by
  alpha and leaves dK, dV unchanged;
* constant V rows give dP - D = 0, hence dQ = dK = 0; dV = P^T dO does not depend on V;
* without the mask, permuting query rows (with their dO rows) permutes dQ and leaves dK,
  dV unchanged; permuting key rows (K and V together) permutes dK, dV and leaves dQ;
* sequences of a batch are independent;
* the tile-wise recomputation (`tiled_attention_bwd_f64`: P rebuilt from the forward's L,
  D taken from the forward's O) equals the untiled derivative for any tile sizes.
"""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import attention_bwd_f64, attention_f64, tiled_attention_bwd_f64

SETTINGS = settings(derandomize=True, max_examples=40, deadline=None, suppress_health_check=[HealthCheck.too_slow])
ATOL = 1e-10


@st.composite
def shapes(draw):
    Hkv = draw(st.integers(1, 2))
    return dict(B=draw(st.integers(1, 2)), Hkv=Hkv, Hq=Hkv * draw(st.integers(1, 3)),
                Nq=draw(st.integers(1, 16)), Nk=draw(st.integers(1, 16)),
                d=draw(st.sampled_from([2, 4, 8])), seed=draw(st.integers(0, 2**31 - 1)),
                scale=draw(st.floats(0.1, 1.5)))


def make(s):
    r = np.random.default_rng(s["seed"])
    q = r.standard_normal((s["B"], s["Hq"], s["Nq"], s["d"]))
    k = r.standard_normal((s["B"], s["Hkv"], s["Nk"], s["d"]))
    v = r.standard_normal((s["B"], s["Hkv"], s["Nk"], s["d"]))
    do = r.standard_normal((s["B"], s["Hq"], s["Nq"], s["d"]))
    return q, k, v, do, r


def allclose(xs, ys, atol=ATOL):
    return all(np.allclose(x, y, rtol=0, atol=atol) for x, y in zip(xs, ys))


@SETTINGS
@given(shapes(), st.booleans())
def test_key_shift_leaves_every_gradient_unchanged(s, causal):
    q, k, v, do, r = make(s)
    c = r.standard_normal(s["d"])
    g1 = attention_bwd_f64(q, k, v, do, causal, s["scale"])
    g2 = attention_bwd_f64(q, k + c, v, do, causal, s["scale"])
    assert allclose(g1, g2, atol=1e-9)


@SETTINGS
@given(shapes(), st.booleans(), st.floats(-2, 2), st.floats(-2, 2))
def test_linear_in_upstream_gradient(s, causal, a, b):
    q, k, v, do1, r = make(s)
    do2 = r.standard_normal(do1.shape)
    g1 = attention_bwd_f64(q, k, v, do1, causal, s["scale"])
    g2 = attention_bwd_f64(q, k, v, do2, causal, s["scale"])
    g3 = attention_bwd_f64(q, k, v, a * do1 + b * do2, causal, s["scale"])
    assert allclose(g3, [a * x + b * y for x, y in zip(g1, g2)])


@SETTINGS
@given(shapes(), st.booleans(), st.floats(0.5, 2.0))
def test_scale_folds_into_queries(s, causal, alpha):
    q, k, v, do, _ = make(s)
    dq1, dk1, dv1 = attention_bwd_f64(q, k, v, do, causal, s["scale"])
    dq2, dk2, dv2 = attention_bwd_f64(alpha * q, k, v, do, causal, s["scale"] / alpha)
    assert allclose([dq2 * alpha, dk2, dv2], [dq1, dk1, dv1], atol=1e-9)


@SETTINGS
@given(shapes(), st.booleans())
def test_constant_values_give_zero_dq_dk(s, causal):
    q, k, v, do, r = make(s)
    dv_any = attention_bwd_f64(q, k, v, do, causal, s["scale"])[2]
    v[:] = r.standard_normal((s["B"], s["Hkv"], 1, s["d"]))      # every V row the same
    dq, dk, dv = attention_bwd_f64(q, k, v, do, causal, s["scale"])
    assert np.allclose(dq, 0, atol=ATOL) and np.allclose(dk, 0, atol=ATOL)
    # dV = P^T dO involves no V at all
    assert np.allclose(dv, dv_any, rtol=0, atol=ATOL)


@SETTINGS
@given(shapes())
def test_query_rows_are_equivariant_without_mask(s):
    q, k, v, do, r = make(s)
    perm = r.permutation(s["Nq"])
    dq1, dk1, dv1 = attention_bwd_f64(q, k, v, do, False, s["scale"])
    dq2, dk2, dv2 = attention_bwd_f64(q[:, :, perm], k, v, do[:, :, perm], False, s["scale"])
    assert allclose([dq2, dk2, dv2], [dq1[:, :, perm], dk1, dv1])


@SETTINGS
@given(shapes(), st.booleans())
def test_batches_are_independent(s, causal):
    q, k, v, do, _ = make(s)
    full = attention_bwd_f64(q, k, v, do, causal, s["scale"])
    for b in range(s["B"]):
        one = attention_bwd_f64(q[b:b + 1], k[b:b + 1], v[b:b + 1], do[b:b + 1], causal, s["scale"])
        assert allclose([x[b:b + 1] for x in full], one)


@SETTINGS
@given(shapes())
def test_key_rows_are_equivariant_without_mask(s):
    """Without the mask, permuting the K and V rows together permutes dK and dV the same
    way and leaves dQ unchanged (this is what catches a row-indexing slip in dK or dV)."""
    q, k, v, do, r = make(s)
    perm = r.permutation(s["Nk"])
    dq1, dk1, dv1 = attention_bwd_f64(q, k, v, do, False, s["scale"])
    dq2, dk2, dv2 = attention_bwd_f64(q, k[:, :, perm], v[:, :, perm], do, False, s["scale"])
    assert allclose([dq2, dk2, dv2], [dq1, dk1[:, :, perm], dv1[:, :, perm]])


@SETTINGS
@given(shapes(), st.booleans(), st.integers(1, 20), st.integers(1, 20))
def test_tiled_recomputation_matches_for_any_tile_sizes(s, causal, Br, Bc):
    """The backward pass as the tiled method runs it: for each key tile and query tile, P
    is recomputed from L and dV, dQ, dK accumulate tile by tile."""
    q, k, v, do, _ = make(s)
    O, L = attention_f64(q, k, v, causal, s["scale"])
    dq, dk, dv = attention_bwd_f64(q, k, v, do, causal, s["scale"])
    g = s["Hq"] // s["Hkv"]
    for b in range(s["B"]):
        dk_t = np.zeros_like(dk[b])
        dv_t = np.zeros_like(dv[b])
        for h in range(s["Hq"]):
            dq_h, dk_h, dv_h = tiled_attention_bwd_f64(q[b, h], k[b, h // g], v[b, h // g], do[b, h],
                                                       O[b, h], L[b, h], causal, s["scale"], Br, Bc)
            assert np.allclose(dq_h, dq[b, h], rtol=0, atol=ATOL)
            dk_t[h // g] += dk_h
            dv_t[h // g] += dv_h
        assert allclose([dk_t, dv_t], [dk[b], dv[b]])
