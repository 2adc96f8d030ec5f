"""Pins for the float64 backward oracle (oracle/backward.py), independent of its formulas:
central finite differences of the forward oracle, hand-worked gradients with exact
closed-form values, closed-form invariants, and the grouped-query sum. CPU only."""
import numpy as np
import pytest

from oracle import attention_bwd_f64, attention_f64


def _rand(shape, rng):
    return rng.standard_normal(shape)


def _loss(q, k, v, do, causal, scale):
    O, _ = attention_f64(q, k, v, causal, scale)
    return float((O * do).sum())


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(4, 4), (3, 5), (5, 3)])
def test_finite_differences(causal, Nq, Nk):
    """d<sum O * dO>/dX by central differences of the forward oracle, every element."""
    rng = np.random.default_rng(11 + 7 * Nq + Nk + causal)
    B, Hq, Hkv, d = 1, 2, 1, 3
    q, k, v = _rand((B, Hq, Nq, d), rng), _rand((B, Hkv, Nk, d), rng), _rand((B, Hkv, Nk, d), rng)
    do = _rand((B, Hq, Nq, d), rng)
    scale = 0.7
    dq, dk, dv = attention_bwd_f64(q, k, v, do, causal, scale)
    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}
            args_m = {"q": q, "k": k, "v": v}
            args_p[name], args_m[name] = xp, xm
            num[idx] = (_loss(args_p["q"], args_p["k"], args_p["v"], do, causal, scale) -
                        _loss(args_m["q"], args_m["k"], args_m["v"], do, causal, scale)) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8, err_msg=f"d{name}")


def test_dv_column_sums_equal_do_sums():
    """Rows of P sum to 1, so sum_j dV_j = sum_i dO_i (every row sees a key)."""
    rng = np.random.default_rng(3)
    q, k, v = _rand((1, 1, 6, 4), rng), _rand((1, 1, 9, 4), rng), _rand((1, 1, 9, 4), rng)
    do = _rand((1, 1, 6, 4), rng)
    for causal in (False, True):
        _, _, dv = attention_bwd_f64(q, k, v, do, causal, 0.5)
        np.testing.assert_allclose(dv[0, 0].sum(axis=0), do[0, 0].sum(axis=0), rtol=1e-12, atol=1e-12)


def test_identical_keys_give_zero_dq():
    """With every key equal, the scores do not depend on q: dQ = 0 and P is uniform."""
    rng = np.random.default_rng(5)
    q = _rand((1, 1, 5, 4), rng)
    k = np.repeat(_rand((1, 1, 1, 4), rng), 7, axis=2)
    v, do = _rand((1, 1, 7, 4), rng), _rand((1, 1, 5, 4), rng)
    dq, _, dv = attention_bwd_f64(q, k, v, do, False, 0.9)
    np.testing.assert_allclose(dq, 0.0, atol=1e-13)
    np.testing.assert_allclose(dv[0, 0], np.repeat(do[0, 0].sum(axis=0, keepdims=True) / 7, 7, axis=0),
                               rtol=1e-12)


def test_grouped_query_heads_sum_into_their_kv_head():
    """Hq = 4 over Hkv = 2 equals Hkv = Hq with K, V duplicated, then summed per group."""
    rng = np.random.default_rng(9)
    q, do = _rand((2, 4, 5, 3), rng), _rand((2, 4, 5, 3), rng)
    k, v = _rand((2, 2, 6, 3), rng), _rand((2, 2, 6, 3), rng)
    dq, dk, dv = attention_bwd_f64(q, k, v, do, True, 0.6)
    kr, vr = np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1)
    dq2, dk2, dv2 = attention_bwd_f64(q, kr, vr, do, True, 0.6)
    np.testing.assert_allclose(dq, dq2, rtol=1e-12)
    np.testing.assert_allclose(dk, dk2.reshape(2, 2, 2, 6, 3).sum(axis=2), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dv, dv2.reshape(2, 2, 2, 6, 3).sum(axis=2), rtol=1e-12, atol=1e-14)


def test_recomputation_identity_matches():
    """The recomputed backward pass uses D_i = sum_d dO_id O_id and P from the saved LSE:
    P_ij = exp(S_ij - LSE_i). Both agree with the oracle's direct quantities."""
    rng = np.random.default_rng(13)
    q, k, v = _rand((1, 1, 4, 3), rng), _rand((1, 1, 6, 3), rng), _rand((1, 1, 6, 3), rng)
    do = _rand((1, 1, 4, 3), rng)
    scale = 0.8
    O, L = attention_f64(q, k, v, True, scale)
    S = scale * q[0, 0] @ k[0, 0].T
    vis = np.arange(6)[None, :] <= (np.arange(4)[:, None] + 2)
    P = np.where(vis, np.exp(S - L[0, 0][:, None]), 0.0)
    D = (do[0, 0] * O[0, 0]).sum(axis=1)
    dS = P * (do[0, 0] @ v[0, 0].T - D[:, None])
    dq, dk, dv = attention_bwd_f64(q, k, v, do, True, scale)
    np.testing.assert_allclose(dq[0, 0], scale * dS @ k[0, 0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dk[0, 0], scale * dS.T @ q[0, 0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dv[0, 0], P.T @ do[0, 0], rtol=1e-12, atol=1e-14)


def test_rows_without_keys_contribute_nothing():
    """Nq > Nk causal: the first Nq - Nk rows see no key; their dQ is 0 and they add nothing."""
    rng = np.random.default_rng(17)
    q, do = _rand((1, 1, 6, 3), rng), _rand((1, 1, 6, 3), rng)
    k, v = _rand((1, 1, 3, 3), rng), _rand((1, 1, 3, 3), rng)
    dq, dk, dv = attention_bwd_f64(q, k, v, do, True, 0.5)
    np.testing.assert_allclose(dq[0, 0, :3], 0.0, atol=0)
    dq2, dk2, dv2 = attention_bwd_f64(q[:, :, 3:], k, v, do[:, :, 3:], True, 0.5)
    np.testing.assert_allclose(dk, dk2, rtol=1e-12)
    np.testing.assert_allclose(dv, dv2, rtol=1e-12)


LN2, LN3 = np.log(2.0), np.log(3.0)


def _hand_worked_cases():
    """Three tiny problems (d = 1, scale = 1/2) whose gradients were derived on paper from
    O = softmax(scale * Q K^T) V. The scores are 0, ln 2, 2 ln 2 or 0, ln 3, so every P is
    rational, and with L = sum(O * dO):
        dV_j = sum_i P_ij dO_i,   dS_ij = P_ij (dO_i v_j - dO_i O_i),
        dQ_i = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i.

    A: q = 2 ln 2, k = (0, 1, 2), v = (7, 0, -7), dO = 2. P = (1/7, 2/7, 4/7), O = -3,
       dS = (20/7, 12/7, -32/7): dQ = -26/7, dK = (20/7, 12/7, -32/7) ln 2,
       dV = (2/7, 4/7, 8/7).
    B: causal, two queries and two keys (bottom-right: row 0 sees key 0 only). Row 0:
       q = 5, dO = 2, P = (1, 0), so dS = 0 and only dV_0 gains 2. Row 1: q = 2 ln 3,
       k = (0, 1), v = (4, 0), dO = 1, P = (1/4, 3/4), O = 1, dS = (3/4, -3/4):
       dQ = (0, -3/8), dK = (3/4, -3/4) ln 3, dV = (9/4, 3/4).
    C: two query heads on one KV head (A's keys and values). Head 0 is A. Head 1: q = 0,
       dO = 3, P = 1/3 each, O = 0, dS = (7, 0, -7): dQ = -7 and no dK. The KV head
       sums both: dK = A's, dV = (9/7, 11/7, 15/7)."""
    col = lambda *x: np.array(x, dtype=np.float64).reshape(-1, 1)
    A = dict(q=col(2 * LN2)[None, None], k=col(0, 1, 2)[None, None], v=col(7, 0, -7)[None, None],
             do=col(2)[None, None], causal=False,
             dq=col(-26 / 7)[None, None], dk=(col(20, 12, -32) / 7 * LN2)[None, None],
             dv=(col(2, 4, 8) / 7)[None, None])
    B = dict(q=col(5, 2 * LN3)[None, None], k=col(0, 1)[None, None], v=col(4, 0)[None, None],
             do=col(2, 1)[None, None], causal=True,
             dq=col(0, -3 / 8)[None, None], dk=(col(3, -3) / 4 * LN3)[None, None],
             dv=col(9 / 4, 3 / 4)[None, None])
    C = dict(q=np.stack([col(2 * LN2), col(0)])[None], k=A["k"], v=A["v"],
             do=np.stack([col(2), col(3)])[None], causal=False,
             dq=np.stack([col(-26 / 7), col(-7)])[None], dk=A["dk"],
             dv=(col(9, 11, 15) / 7)[None, None])
    return {"A": A, "B": B, "C": C}


def _hand_worked_matches(bwd):
    """True if `bwd` (a replacement for the per-head gradient) reproduces every hand-worked
    gradient to 1e-12."""
    import oracle.backward as ob
    saved = ob._head_bwd
    ob._head_bwd = bwd
    try:
        for c in _hand_worked_cases().values():
            got = ob.attention_bwd_f64(c["q"], c["k"], c["v"], c["do"], c["causal"], 0.5)
            for g, want in zip(got, (c["dq"], c["dk"], c["dv"])):
                if g.shape != want.shape or not np.allclose(g, want, rtol=0, atol=1e-12):
                    return False
    finally:
        ob._head_bwd = saved
    return True


def test_hand_worked_gradients():
    import oracle.backward as ob
    assert _hand_worked_matches(ob._head_bwd)


def _fd_matches(bwd, causal):
    """True if `bwd` (a replacement for the per-head gradient) agrees with finite
    differences of the forward oracle on a small problem."""
    import oracle.backward as ob
    rng = np.random.default_rng(21)
    q, k, v = _rand((1, 1, 4, 3), rng), _rand((1, 1, 5, 3), rng), _rand((1, 1, 5, 3), rng)
    do = _rand((1, 1, 4, 3), rng)
    saved = ob._head_bwd
    ob._head_bwd = bwd
    try:
        dq, dk, dv = ob.attention_bwd_f64(q, k, v, do, causal, 0.7)
    finally:
        ob._head_bwd = saved
    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            a = {"q": q, "k": k, "v": v}
            b = {"q": q, "k": k, "v": v}
            a[name], b[name] = xp, xm
            num = (_loss(a["q"], a["k"], a["v"], do, causal, 0.7) - _loss(b["q"], b["k"], b["v"], do, causal, 0.7)) / (2 * eps)
            if not np.isclose(g[idx], num, rtol=1e-6, atol=1e-8):
                return False
    return True


def test_mutants_fail_the_finite_difference_pin():
    """Plausible mistakes in the gradient formulas are caught by the finite-difference pin
    and by the hand-worked one."""
    import oracle.backward as ob
    right = ob._head_bwd

    def drop_d(Q, K, V, dO, vis, scale):              # dS = P * dP (the D term dropped)
        S = np.where(vis, scale * (Q @ K.T), -np.inf)
        P = np.exp(S - S.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        dS = P * (dO @ V.T)
        return scale * dS @ K, scale * dS.T @ Q, P.T @ dO

    def no_scale_dq(Q, K, V, dO, vis, scale):          # dQ without the scale factor
        dQ, dK, dV = right(Q, K, V, dO, vis, scale)
        return dQ / scale, dK, dV

    def misindexed_dk(Q, K, V, dO, vis, scale):        # dK rows in reverse key order
        dQ, dK, dV = right(Q, K, V, dO, vis, scale)
        return dQ, np.flipud(dK), dV

    assert _fd_matches(right, True) and _hand_worked_matches(right)
    for bad in (drop_d, no_scale_dq, misindexed_dk):
        assert not _fd_matches(bad, True), bad.__name__
        assert not _hand_worked_matches(bad), bad.__name__
