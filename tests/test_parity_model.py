"""CPU checks of the rounding models that set the backward and E4M3 tolerances
(`bwd_head_terms` / `assert_close_bwd` and `fp8_sigma` / `assert_close_fp8` in
`tests/parity.py`).

Each test emulates, in float64, the roundings that the kernels perform and nothing else:
every product and sum is exact here, and the values the kernels hold in 16 bits (or in
E4M3) are rounded to that format by torch's conversion (round to nearest even). A model
that is right must then

* accept the emulated result: every element within the 6 sigma bound (the same assertion
  the GPU tests make), and
* be tight: the emulated RMS error is a fixed fraction of the model's RMS sigma, between
  0.5 and 0.9. Uniform relative error on [-u, u] overstates round-to-nearest-even by about
  sqrt(2) in RMS, so about 0.7 is expected. A model whose variances are 4x too large or
  too small falls outside the range, and one that drops the dS or the D term puts
  elements past 6 sigma. The E4M3 model's window starts at 0.4: the largest P of a row is
  2^4 exactly and carries no rounding error, which the model still counts, and causal rows
  with few keys are dominated by that term.

The rounding points emulated:

* backward: the forward's 16-bit P (operand of P.V) and 16-bit O; P recomputed from the
  LSE; 16-bit P as the operand of dV = P^T dO; D = rowsum(dO * O) from the 16-bit O;
  dS = P * (dP - D) rounded to 16 bits as the operand of dQ and dK; each gradient rounded
  to 16 bits at the end (a KV head's dK, dV summed over its query heads first);
* E4M3: P = 2^(log2(e) * (s - m) + 4) (the kernel's offset keeps P normal), rounded to
  E4M3 as the operand of P.V; the row sum from P before rounding; O rounded to bf16;
* 16-bit forward: P rounded to 16 bits as the operand of P.V, the row sum from P before
  rounding, O rounded to 16 bits. Its tolerances are fixed numbers, not a model; the
  emulated errors must stay inside them with room to spare (max-abs at most 3/4 of the
  bound), so that a kernel with these roundings passes for a reason, not by luck;
* decode: per split of 1024 keys (d = 128, tensor cores) P rounded to 16 bits as the P.V
  operand and the split's row sum from P before rounding; the fp32 partials merged by
  their LSEs; O rounded to 16 bits. At d = 64 (CUDA cores) P stays fp32 and only O is
  rounded. Same fixed tolerances, same room.
"""
import math

import numpy as np
import pytest
import torch

from oracle import (attention_bwd_f64, attention_f64, attention_fp8_f64, decode_f64, e4m3_to_f64,
                    visible_mask)
from tests.parity import (LSE_REL, MAX_ABS, RMS_TOL, assert_close_bwd, assert_close_fp8,
                          bwd_head_terms, fp8_sigma, metrics, to_f64)
from workloads import make_decode_inputs, make_fp8_inputs, make_fwd_inputs

TIGHT = (0.5, 0.9)
TIGHT_FP8 = (0.4, 0.9)
DT = {"fp16": torch.float16, "bf16": torch.bfloat16}


def r16(x: np.ndarray, dtype: str) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x)).to(DT[dtype]).double().numpy()


def e4m3(x: np.ndarray) -> np.ndarray:
    codes = torch.from_numpy(np.ascontiguousarray(x)).float().to(torch.float8_e4m3fn)
    return e4m3_to_f64(codes.view(torch.uint8))


def emulate_bwd_head(Q, K, V, dO, vis, scale, dtype):
    """(dQ, dK-contribution, dV-contribution) of one query head before output rounding."""
    S = np.where(vis, scale * (Q @ K.T), -np.inf)
    m = S.max(axis=1)
    has = np.isfinite(m)
    E = np.zeros_like(S)
    E[has] = np.exp(S[has] - m[has, None])
    l = E.sum(axis=1)
    O = np.zeros_like(Q)
    O[has] = r16((r16(E[has], dtype) @ V) / l[has, None], dtype)      # the forward's O
    lse = np.full(len(m), -np.inf)
    lse[has] = m[has] + np.log(l[has])
    P = np.zeros_like(S)
    P[has] = np.exp(S[has] - lse[has, None])                           # recomputed P
    dV = r16(P, dtype).T @ dO
    dP = dO @ V.T
    D = (dO * O).sum(axis=1)
    dS = r16(P * (dP - D[:, None]), dtype)
    return scale * (dS @ K), scale * (dS.T @ Q), dV


def bwd_case(B, Hq, Hkv, N, d, dtype, causal, seed):
    q, k, v = make_fwd_inputs(B, Hq, Hkv, N, N, d, dtype, seed)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(seed + 1)).to(q.dtype)
    q, k, v, dout = to_f64(q), to_f64(k), to_f64(v), to_f64(dout)
    scale = 1.0 / math.sqrt(d)
    vis = visible_mask(np.arange(N), N, N, causal)
    ref = attention_bwd_f64(q, k, v, dout, causal, scale)
    g = Hq // Hkv
    stats = []
    for b in range(B):
        for kh in range(Hkv):
            dk = np.zeros((N, d))
            dv = np.zeros((N, d))
            var_k = np.zeros((N, d))
            var_v = np.zeros((N, d))
            for h in range(kh * g, (kh + 1) * g):
                dq_h, dk_h, dv_h = emulate_bwd_head(q[b, h], k[b, kh], v[b, kh], dout[b, h], vis,
                                                    scale, dtype)
                dk += dk_h
                dv += dv_h
                t = bwd_head_terms(q[b, h], k[b, kh], v[b, kh], dout[b, h], vis, scale, dtype)
                var_k += t[4]
                var_v += t[5]
                stats.append(assert_close_bwd(r16(dq_h, dtype), ref[0][b, h], t[3], dtype,
                                              f"dq b{b} h{h}"))
            stats.append(assert_close_bwd(r16(dk, dtype), ref[1][b, kh], var_k, dtype, f"dk b{b} kh{kh}"))
            stats.append(assert_close_bwd(r16(dv, dtype), ref[2][b, kh], var_v, dtype, f"dv b{b} kh{kh}"))
    return stats


@pytest.mark.parametrize("d,dtype", [(64, "fp16"), (128, "bf16")])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_model_accepts_and_is_tight(d, dtype, causal):
    stats = bwd_case(1, 4, 2, 256, d, dtype, causal, seed=d + causal)
    ratios = [s["rms_err_over_rms_sigma"] for s in stats]
    assert TIGHT[0] <= min(ratios) and max(ratios) <= TIGHT[1], ratios
    assert max(s["max_err_over_sigma"] for s in stats) <= 6.0


def emulate_fp8(q8, k8, v8, dq, dk, dv, causal, scale):
    """O (bf16-rounded) of the E4M3 path for every head, float64 [B, Hq, Nq, d]."""
    Q, K, V = e4m3_to_f64(q8) * dq, e4m3_to_f64(k8) * dk, e4m3_to_f64(v8) * dv
    B, Hq, Nq, d = Q.shape
    Hkv, Nk = K.shape[1], K.shape[2]
    vis = visible_mask(np.arange(Nq), Nq, Nk, causal)
    out = np.zeros((B, Hq, Nq, d))
    for b in range(B):
        for h in range(Hq):
            kh = h // (Hq // Hkv)
            S = np.where(vis, scale * (Q[b, h] @ K[b, kh].T), -np.inf)
            m = S.max(axis=1)
            P = np.exp2(np.log2(np.e) * (S - m[:, None]) + 4.0)
            l = P.sum(axis=1)
            out[b, h] = r16((e4m3(P) @ V[b, kh]) / l[:, None], "bf16")
    return out


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_model_accepts_and_is_tight(causal):
    q8, k8, v8, dq, dk, dv = make_fp8_inputs(1, 2, 1, 384, 384, 128, seed=7 + causal)
    scale = 1.0 / math.sqrt(128)
    O, L = attention_fp8_f64(q8, k8, v8, dq, dk, dv, causal, scale)
    got = emulate_fp8(q8, k8, v8, dq, dk, dv, causal, scale)
    Q, K, V = e4m3_to_f64(q8) * dq, e4m3_to_f64(k8) * dk, e4m3_to_f64(v8) * dv
    for h in range(2):
        sigma = fp8_sigma(Q[0, h], K[0, 0], V[0, 0], causal, scale, np.arange(384), 384)
        s = assert_close_fp8(torch.from_numpy(got[0, h]), None, O[0, h], L[0, h], sigma,
                             f"fp8 h{h}")
        ratio = s["rms"] / s["rms_sigma"]
        assert TIGHT_FP8[0] <= ratio <= TIGHT_FP8[1], s


def emulate_fwd_head(Q, K, V, vis, scale, dtype):
    """O (16-bit-rounded) and LSE of one head with the 16-bit kernel's roundings."""
    S = np.where(vis, scale * (Q @ K.T), -np.inf)
    m = S.max(axis=1)
    E = np.exp(S - m[:, None])
    l = E.sum(axis=1)
    return r16((r16(E, dtype) @ V) / l[:, None], dtype), m + np.log(l)


@pytest.mark.parametrize("d,dtype", [(64, "fp16"), (128, "bf16")])
@pytest.mark.parametrize("causal", [False, True])
def test_forward_roundings_fit_the_fixed_tolerances(d, dtype, causal):
    N = 2048
    q, k, v = make_fwd_inputs(1, 1, 1, N, N, d, dtype, seed=d + 2 * causal)
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    scale = 1.0 / math.sqrt(d)
    O, L = attention_f64(q, k, v, causal, scale)
    got, lse = emulate_fwd_head(q[0, 0], k[0, 0], v[0, 0], visible_mask(np.arange(N), N, N, causal),
                                scale, dtype)
    m = metrics(got, lse, O[0, 0], L[0, 0])
    assert m["max_abs"] <= 0.75 * MAX_ABS[dtype], m
    assert m["rms"] <= 0.5 * RMS_TOL and m["lse_rel"] <= 0.01 * LSE_REL, m


def emulate_decode_head(q, K, V, split, round_p, dtype):
    """O (16-bit-rounded) and LSE of one decode row: splits of `split` keys, each with its
    own maximum (P rounded to 16 bits when round_p), merged by the splits' LSEs."""
    parts = []
    for s0 in range(0, K.shape[0], split):
        sc = (K[s0:s0 + split] @ q)
        m = sc.max()
        e = np.exp(sc - m)
        pv = (r16(e, dtype) if round_p else e) @ V[s0:s0 + split]
        parts.append((pv / e.sum(), m + np.log(e.sum())))
    lse = np.logaddexp.reduce([l for _, l in parts])
    return r16(sum(np.exp(l - lse) * o for o, l in parts), dtype), lse


@pytest.mark.parametrize("d,dtype,round_p", [(128, "bf16", True), (64, "fp16", False)])
def test_decode_roundings_fit_the_fixed_tolerances(d, dtype, round_p):
    lens, q, kc, vc = make_decode_inputs(4, 32, 8, 4096, d, dtype, 512, 4096, seed=d)
    q, kc, vc = to_f64(q), to_f64(kc), to_f64(vc)
    scale = 1.0 / math.sqrt(d)
    O, L = decode_f64(q, kc, vc, lens, scale)
    got = np.zeros_like(O)
    lse = np.zeros_like(L)
    for b in range(4):
        n = int(lens[b])
        for h in range(32):
            got[b, h], lse[b, h] = emulate_decode_head(scale * q[b, h], kc[b, h // 4, :n],
                                                       vc[b, h // 4, :n], 1024, round_p, dtype)
    m = metrics(got, lse, O, L)
    assert m["max_abs"] <= 0.75 * MAX_ABS[dtype], m
    assert m["rms"] <= 0.5 * RMS_TOL and m["lse_rel"] <= 0.01 * LSE_REL, m
