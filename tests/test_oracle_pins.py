"""CPU checks that pin the float64 oracle to facts outside itself."""
import math

import numpy as np
import pytest
import torch

from oracle import attention_f64, attention_rows_f64, decode_f64, tiled_attention_f64
from tests import oracle_pins
from workloads import make_decode_inputs, make_fwd_inputs


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(attention_f64)


@pytest.mark.parametrize("Br,Bc", [(1, 1), (3, 3), (16, 16), (128, 128), (3, 16), (16, 3)])
@pytest.mark.parametrize("Nq,Nk,causal", [(1, 1, False), (37, 37, True), (130, 130, True),
                                          (300, 300, True), (50, 171, True), (171, 50, True),
                                          (129, 257, False)])
def test_tiled_online_softmax_equals_untiled(Br, Bc, Nq, Nk, causal):
    """The exactness claim: tiled online softmax (running max and normaliser) gives the
    untiled result to 1e-12, including lengths that are not tile multiples."""
    r = np.random.default_rng(Nq * 1000 + Nk)
    Q = r.standard_normal((Nq, 8))
    K = r.standard_normal((Nk, 8))
    V = r.standard_normal((Nk, 8))
    O1, L1 = tiled_attention_f64(Q, K, V, causal, 0.4, Br, Bc)
    O2, L2 = attention_f64(Q[None, None], K[None, None], V[None, None], causal, 0.4)
    assert np.allclose(O1, O2[0, 0], rtol=0, atol=1e-12)
    fin = np.isfinite(L2[0, 0])
    assert np.array_equal(np.isfinite(L1), fin)
    assert np.allclose(L1[fin], L2[0, 0][fin], rtol=0, atol=1e-12)


def test_tiled_satisfies_pins():
    """The tiled restatement passes the same pins, wrapped per head."""
    def tiled(q, k, v, causal, scale):
        B, Hq, Nq, d = q.shape
        g = Hq // k.shape[1]
        O = np.zeros((B, Hq, Nq, d))
        L = np.zeros((B, Hq, Nq))
        for b in range(B):
            for h in range(Hq):
                O[b, h], L[b, h] = tiled_attention_f64(q[b, h], k[b, h // g], v[b, h // g],
                                                       causal, scale, 4, 5)
        return O, L
    for pin in (oracle_pins.pin_golden, oracle_pins.pin_brute_force, oracle_pins.pin_zero_query,
                oracle_pins.pin_causal_first_row):
        pin(tiled)


def test_rows_subset_matches_full():
    q, k, v = make_fwd_inputs(1, 4, 2, 300, 300, 64, "bf16", seed=3)
    O, L = attention_f64(q, k, v, True, 0.125)
    rows = [0, 1, 127, 128, 255, 299]
    for h in range(4):
        o, l = attention_rows_f64(q, k, v, True, 0.125, 0, h, rows)
        assert np.array_equal(o, O[0, h, rows]) and np.array_equal(l, L[0, h, rows])


def test_decode_equals_single_row_attention():
    """Decode = the attention definition with Nq = 1, non-causal, over cache[:kv_len]."""
    kv_lens, q, kc, vc = make_decode_inputs(3, 8, 2, 64, 64, "bf16", 1, 64, seed=5,
                                            kv_lens=torch.tensor([1, 37, 64]))
    O, L = decode_f64(q, kc, vc, kv_lens, 0.125)
    for b in range(3):
        n = int(kv_lens[b])
        Ob, Lb = attention_f64(q[b][None, :, None, :], kc[b][None, :, :n], vc[b][None, :, :n],
                               False, 0.125)
        assert np.allclose(O[b], Ob[0, :, 0], rtol=0, atol=1e-13)
        assert np.allclose(L[b], Lb[0, :, 0], rtol=0, atol=1e-13)


def test_decode_zero_length_row():
    kv_lens, q, kc, vc = make_decode_inputs(2, 4, 1, 16, 64, "fp16", 1, 16, seed=6,
                                            kv_lens=torch.tensor([0, 16]))
    O, L = decode_f64(q, kc, vc, kv_lens, 0.125)
    assert np.all(O[0] == 0) and np.all(L[0] == -np.inf) and np.all(np.isfinite(L[1]))


def test_lse_reconstructs_output():
    """O = sum_j exp(s_ij - LSE_i) V_j with the oracle's LSE (LSE carries the normaliser)."""
    q, k, v = make_fwd_inputs(1, 2, 2, 40, 40, 16, "fp16", seed=7)
    O, L = attention_f64(q, k, v, True, 0.25)
    qf, kf, vf = (x.double().numpy() for x in (q, k, v))
    for h in range(2):
        S = 0.25 * qf[0, h] @ kf[0, h].T
        S[np.triu_indices(40, 1)] = -np.inf
        assert np.allclose(np.exp(S - L[0, h, :, None]) @ vf[0, h], O[0, h], atol=1e-12, rtol=0)


def test_inputs_upcast_exactly():
    """16-bit inputs reach the oracle unchanged (the upcast is exact)."""
    q, k, v = make_fwd_inputs(1, 1, 1, 8, 8, 64, "bf16", seed=8)
    O, L = attention_f64(q, k, v, True, 0.125)
    assert np.array_equal(O[0, 0, 0], v[0, 0, 0].float().double().numpy())
    assert math.isclose(L[0, 0, 0], 0.125 * float((q[0, 0, 0].double() @ k[0, 0, 0].double())),
                        rel_tol=0, abs_tol=1e-15)
