"""GPU parity of fa_fwd_fp8 (E4M3 Q, K, V) with the float64 oracle on the descaled inputs.
The tolerance is the E4M3 rounding model of P stated in tests/parity.py (6 sigma per
output plus bf16 output rounding); LSE is held to the 16-bit path's 1e-4 relative."""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_28_b200 as fa
from oracle import attention_fp8_f64, attention_fp8_rows_f64, e4m3_to_f64
from tests.parity import assert_close_fp8, fp8_sigma, sample_rows
from workloads import WORKLOADS, make_fp8_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def sigma_full(q8, k8, v8, dq, dk, dv, causal, scale):
    B, Hq, Nq, d = q8.shape
    Hkv = k8.shape[1]
    out = np.zeros((B, Hq, Nq, d))
    for b in range(B):
        for h in range(Hq):
            kh = h // (Hq // Hkv)
            out[b, h] = fp8_sigma(e4m3_to_f64(q8[b, h]) * dq, e4m3_to_f64(k8[b, kh]) * dk,
                                  e4m3_to_f64(v8[b, kh]) * dv, causal, scale, np.arange(Nq), Nq)
    return out


def run(q8, k8, v8, dq, dk, dv, causal, scale):
    o, lse = fa.fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), dq, dk, dv, causal=causal,
                        scale=scale)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    return o.cpu(), lse.cpu()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(128, 128), (300, 77), (77, 300), (1, 513), (1024, 1024),
                                   (600, 1500)])
def test_fp8_shapes(causal, Nq, Nk):
    B, Hq, Hkv, d = 2, 4, 2, 128
    q8, k8, v8, dq, dk, dv = make_fp8_inputs(B, Hq, Hkv, Nq, Nk, d, seed=Nq + 3 * Nk)
    scale = 1.0 / math.sqrt(d)
    o, lse = run(q8, k8, v8, dq, dk, dv, causal, scale)
    O, L = attention_fp8_f64(q8, k8, v8, dq, dk, dv, causal, scale)
    sig = sigma_full(q8, k8, v8, dq, dk, dv, causal, scale)
    assert_close_fp8(o, lse, O, L, sig, f"fp8 c{causal} Nq{Nq} Nk{Nk}")


def test_fp8_peaked_rows_and_rescales():
    """Scores that grow along the keys force rescales of the running maximum, and a few
    dominant keys per row make the softmax peaked (few terms in the rounding sum)."""
    B, Hq, Hkv, N, d = 1, 2, 1, 700, 128
    q8, k8, v8, dq, dk, dv = make_fp8_inputs(B, Hq, Hkv, N, N, d, seed=91)
    kf = e4m3_to_f64(k8) * dk
    ramp = np.linspace(0.2, 3.0, N)[None, None, :, None]
    k_new = torch.from_numpy((kf * ramp / dk).astype(np.float32))
    amax = float(k_new.abs().max())
    k8 = (k_new * (448.0 / amax)).to(torch.float8_e4m3fn).view(torch.uint8)
    dk = dk * amax / 448.0
    scale = 2.0 / math.sqrt(d)
    for causal in (False, True):
        o, lse = run(q8, k8, v8, dq, dk, dv, causal, scale)
        O, L = attention_fp8_f64(q8, k8, v8, dq, dk, dv, causal, scale)
        sig = sigma_full(q8, k8, v8, dq, dk, dv, causal, scale)
        assert_close_fp8(o, lse, O, L, sig, f"fp8 peaked c{causal}")


def test_fp8_gqa8k_sampled_rows():
    """The causal GQA workload's shape (Hq 32, Hkv 8, 8192 tokens, d 128) in E4M3."""
    w = WORKLOADS["gqa8k"]
    q8, k8, v8, dq, dk, dv = make_fp8_inputs(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, seed=w.seed)
    o, lse = run(q8, k8, v8, dq, dk, dv, True, w.scale)
    rows = sample_rows(w.N, 48, seed=8)
    for h in (0, 5, 18, 31):
        O, L = attention_fp8_rows_f64(q8, k8, v8, dq, dk, dv, True, w.scale, 0, h, rows)
        kh = h // (w.Hq // w.Hkv)
        sig = fp8_sigma(e4m3_to_f64(q8[0, h])[rows] * dq, e4m3_to_f64(k8[0, kh]) * dk,
                        e4m3_to_f64(v8[0, kh]) * dv, True, w.scale, rows, w.N)
        assert_close_fp8(o[0, h, rows], lse[0, h, rows], O, L, sig, f"fp8 gqa8k h{h}")
