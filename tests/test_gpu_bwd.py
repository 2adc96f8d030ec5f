"""GPU parity of fa_bwd (dQ, dK, dV by recomputation) with the float64 backward oracle.

Tolerances are relative to each gradient's scale. The gradients pass through 16-bit P and
dS operands of the tensor-core products (as the forward's P does) and are written in 16
bits, so their error is a few units of the 16-bit rounding: relative RMS <= 1.5e-2 (bf16)
/ 4e-3 (fp16), relative max <= 4e-2 / 1.2e-2."""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_28_b200 as fa
from oracle import attention_bwd_f64
from tests.parity import to_f64
from workloads import make_fwd_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TOL = {"bf16": (1.5e-2, 4e-2), "fp16": (4e-3, 1.2e-2)}


def check_bwd(B, Hq, Hkv, Nq, Nk, d, dtype, causal, seed=0):
    q, k, v = make_fwd_inputs(B, Hq, Hkv, Nq, Nk, d, dtype, seed)
    g = torch.Generator().manual_seed(seed + 1)
    dout = torch.randn(q.shape, generator=g).to(q.dtype)
    scale = 1.0 / math.sqrt(d)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), dout.to(DEV)
    o, lse = fa.fwd(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, lse, dod, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    ref = attention_bwd_f64(q, k, v, dout, causal, scale)
    rms_tol, max_tol = TOL[dtype]
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        got = to_f64(got.cpu())
        assert np.all(np.isfinite(got)), name
        scale_rms = math.sqrt(float(np.mean(want ** 2))) + 1e-30
        err = got - want
        rel_rms = math.sqrt(float(np.mean(err ** 2))) / scale_rms
        rel_max = float(np.max(np.abs(err))) / (float(np.max(np.abs(want))) + 1e-30)
        assert rel_rms <= rms_tol and rel_max <= max_tol, \
            f"{name} B{B} Hq{Hq} Hkv{Hkv} Nq{Nq} Nk{Nk} d{d} {dtype} c{causal}: rel_rms {rel_rms:.2e} rel_max {rel_max:.2e}"


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 200, 384])
def test_square(d, dtype, causal, N):
    check_bwd(1, 2, 2, N, N, d, dtype, causal, seed=N + d)


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (8, 1)])
@pytest.mark.parametrize("causal", [False, True])
def test_grouped_query_heads(Hq, Hkv, causal):
    """dK and dV of a KV head sum over every query head that reads it."""
    check_bwd(2, Hq, Hkv, 256, 256, 128, "bf16", causal, seed=Hq * 10 + Hkv)


@pytest.mark.parametrize("Nq,Nk", [(128, 300), (300, 128), (77, 513)])
@pytest.mark.parametrize("causal", [False, True])
def test_rectangular(Nq, Nk, causal):
    """Nq != Nk with bottom-right causal alignment; Nq > Nk has rows without keys."""
    check_bwd(1, 4, 2, Nq, Nk, 64, "fp16", causal, seed=Nq + 3 * Nk)


def test_mha2k_workload_sampled_heads():
    """The full causal B=8 H=12 N=2048 d=64 fp16 backward pass; two (batch, head) problems
    checked element by element against the oracle (each head is independent here)."""
    from workloads import WORKLOADS
    w = WORKLOADS["mha2k"]
    q, k, v = make_fwd_inputs(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, w.seed)
    g = torch.Generator().manual_seed(w.seed + 1)
    dout = torch.randn(q.shape, generator=g).to(q.dtype)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), dout.to(DEV)
    o, lse = fa.fwd(qd, kd, vd, causal=True, scale=w.scale)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, lse, dod, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    rms_tol, max_tol = TOL[w.dtype]
    for b, h in ((0, 0), (w.B - 1, w.Hq - 1)):
        sl = slice(b, b + 1), slice(h, h + 1)
        ref = attention_bwd_f64(q[sl], k[sl], v[sl], dout[sl], True, w.scale)
        for name, got, want in zip(("dq", "dk", "dv"), (dq[sl], dk[sl], dv[sl]), ref):
            got = to_f64(got.cpu())
            err = got - want
            rel_rms = math.sqrt(float(np.mean(err ** 2))) / math.sqrt(float(np.mean(want ** 2)))
            rel_max = float(np.max(np.abs(err))) / float(np.max(np.abs(want)))
            assert rel_rms <= rms_tol and rel_max <= max_tol, f"{name} b{b} h{h}: {rel_rms:.2e} {rel_max:.2e}"
