"""GPU parity of fa_bwd (dQ, dK, dV by recomputation) with the float64 backward oracle.

Tolerances come from a rounding model of the kernels' 16-bit operands (`tests/parity.py`,
`bwd_head_terms` and `assert_close_bwd`): the 16-bit P of dV = P^T dO, the 16-bit dS of
dQ and dK, the forward's 16-bit O that D is taken from, and the output rounding, each an
independent relative error within the 16-bit unit roundoff. Every element must lie within
6 sigma of the oracle, and the RMS error within the model's RMS sigma."""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_28_b200 as fa
from oracle import attention_bwd_f64, visible_mask
from tests.parity import assert_close_bwd, bwd_head_terms, to_f64
from workloads import make_fwd_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def model_vars(q, k, v, dout, causal, scale, dtype, b, heads):
    """Error-model variances of dQ for query heads `heads` of batch b, and of dK, dV for
    the KV heads those heads read (summed over the heads of each group that are listed)."""
    Hq, Nq = q.shape[1], q.shape[2]
    Hkv, Nk = k.shape[1], k.shape[2]
    g = Hq // Hkv
    vis = visible_mask(np.arange(Nq), Nq, Nk, causal)
    var_q, var_k, var_v = {}, {}, {}
    for h in heads:
        kh = h // g
        t = bwd_head_terms(to_f64(q[b, h]), to_f64(k[b, kh]), to_f64(v[b, kh]), to_f64(dout[b, h]),
                           vis, scale, dtype)
        var_q[h] = t[3]
        var_k[kh] = var_k.get(kh, 0.0) + t[4]
        var_v[kh] = var_v.get(kh, 0.0) + t[5]
    return var_q, var_k, var_v


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
    dq, dk, dv = to_f64(dq.cpu()), to_f64(dk.cpu()), to_f64(dv.cpu())
    what = f"B{B} Hq{Hq} Hkv{Hkv} Nq{Nq} Nk{Nk} d{d} {dtype} c{causal}"
    for b in range(B):
        var_q, var_k, var_v = model_vars(q, k, v, dout, causal, scale, dtype, b, range(Hq))
        for h in range(Hq):
            assert_close_bwd(dq[b, h], ref[0][b, h], var_q[h], dtype, f"dq b{b} h{h} {what}")
        for kh in range(Hkv):
            assert_close_bwd(dk[b, kh], ref[1][b, kh], var_k[kh], dtype, f"dk b{b} kh{kh} {what}")
            assert_close_bwd(dv[b, kh], ref[2][b, kh], var_v[kh], dtype, f"dv b{b} kh{kh} {what}")


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


@pytest.mark.parametrize("B,Hq,Hkv,N,d,dtype,causal", [
    (2, 8, 2, 1000, 64, "fp16", True),     # 16 key tiles per dQ tile: the ring wraps
    (1, 4, 1, 777, 128, "bf16", False),    # odd step counts, 4 query heads per KV head
])
def test_longer_ragged_sequences(B, Hq, Hkv, N, d, dtype, causal):
    """Many steps per CTA with a ragged last tile: the dQ pass alternates its two dP
    buffers and loads V ahead of K through several turns of the ring; the dK/dV pass runs
    its two elementwise passes across the query heads of a group."""
    check_bwd(B, Hq, Hkv, N, N, d, dtype, causal, seed=N + Hq)


@pytest.mark.parametrize("d", [64, 128])
def test_bounded_wait_reports_timeout_and_context_survives(d):
    """Test hook: neither pass loads its resident tiles, so every wait on them runs out
    after 20 ms; the kernels record FA_ERR_DEVICE_TIMEOUT, drain and return, and the next
    call is correct."""
    dtype = "fp16" if d == 64 else "bf16"
    q, k, v = make_fwd_inputs(1, 2, 1, 256, 256, d, dtype, seed=31 + d)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(32)).to(q.dtype)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), dout.to(DEV)
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.fwd(qd, kd, vd, causal=True, scale=scale)
    torch.cuda.synchronize()
    assert fa.device_status(clear=True) == fa.FA_OK
    fa.set_wait_timeout_ns(20_000_000)
    fa.debug_skip_q_load(True)
    try:
        fa.bwd(qd, kd, vd, o, lse, dod, causal=True, scale=scale)
        status = fa.device_status(clear=True)
    finally:
        fa.debug_skip_q_load(False)
        fa.set_wait_timeout_ns(0)
    assert status == fa.FA_ERR_DEVICE_TIMEOUT
    check_bwd(1, 2, 1, 256, 256, d, dtype, True, seed=31 + d)


def full_size_case(name, checks):
    """The workload's full backward pass in one call; `checks` = [(b, kv_head)]: dK and dV
    of each listed KV head (all its query heads) and dQ of those query heads against the
    oracle, run per KV group on slices of the inputs (groups are independent)."""
    from workloads import WORKLOADS
    w = WORKLOADS[name]
    q, k, v = make_fwd_inputs(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, w.seed)
    gen = torch.Generator().manual_seed(w.seed + 1)
    dout = torch.randn(q.shape, generator=gen).to(q.dtype)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), dout.to(DEV)
    o, lse = fa.fwd(qd, kd, vd, causal=w.causal, scale=w.scale)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, lse, dod, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    del qd, kd, vd, dod, o, lse
    g = w.Hq // w.Hkv
    out = []
    for b, kh in checks:
        hs = slice(kh * g, (kh + 1) * g)
        sl_q = (slice(b, b + 1), hs)
        sl_k = (slice(b, b + 1), slice(kh, kh + 1))
        ref = attention_bwd_f64(q[sl_q], k[sl_k], v[sl_k], dout[sl_q], w.causal, w.scale)
        var_q, var_k, var_v = model_vars(q[sl_q], k[sl_k], v[sl_k], dout[sl_q], w.causal, w.scale,
                                         w.dtype, 0, range(g))
        for i in range(g):
            out.append(assert_close_bwd(to_f64(dq[b, kh * g + i].cpu()), ref[0][0, i], var_q[i],
                                        w.dtype, f"{name} dq b{b} h{kh * g + i}"))
        out.append(assert_close_bwd(to_f64(dk[b, kh].cpu()), ref[1][0, 0], var_k[0], w.dtype,
                                    f"{name} dk b{b} kh{kh}"))
        out.append(assert_close_bwd(to_f64(dv[b, kh].cpu()), ref[2][0, 0], var_v[0], w.dtype,
                                    f"{name} dv b{b} kh{kh}"))
    return out


def test_mha2k_workload_sampled_heads():
    """The full causal B=8 H=12 N=2048 d=64 fp16 backward pass; the first and the last
    (batch, head) problems checked element by element (each head is its own group here)."""
    stats = full_size_case("mha2k", [(0, 0), (7, 11)])
    print("mha2k bwd:", stats)


def test_gqa8k_workload_sampled_groups():
    """The full causal B=1 Hq=32 Hkv=8 N=8192 d=128 bf16 backward pass; KV heads 0 and 7
    with their four query heads each, every element of dQ, dK and dV."""
    stats = full_size_case("gqa8k", [(0, 0), (0, 7)])
    print("gqa8k bwd:", stats)
