"""GPU parity of fa_decode (through the C ABI) against the float64 CPU oracle."""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_28_b200 as fa
from oracle import decode_f64
from tests.parity import assert_close
from workloads import WORKLOADS, make_decode_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def run_decode(kv_lens, q, kc, vc, scale, workspace=None):
    o, lse = fa.decode(q.to(DEV), kc.to(DEV), vc.to(DEV), kv_lens.to(DEV), scale=scale,
                       workspace=workspace)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    return o.cpu(), lse.cpu()


def check(B, Hq, Hkv, cache, d, dtype, lens, seed=0):
    kv_lens, q, kc, vc = make_decode_inputs(B, Hq, Hkv, cache, d, dtype, 1, cache, seed,
                                            kv_lens=torch.tensor(lens))
    scale = 1.0 / math.sqrt(d)
    o, lse = run_decode(kv_lens, q, kc, vc, scale)
    O, L = decode_f64(q, kc, vc, kv_lens, scale)
    return assert_close(o, lse, O, L, dtype, f"decode B{B} Hq{Hq} Hkv{Hkv} d{d} {dtype} {lens}",
                        strict=False)


def test_decode_workload_full():
    """B=64, Hq=32, Hkv=8, d=128 bf16, kv_len ~ U[512, 4096] from seed 0: every output."""
    w = WORKLOADS["decode"]
    kv_lens, q, kc, vc = make_decode_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.dtype, w.kv_len_lo,
                                            w.kv_len_hi, w.seed)
    o, lse = run_decode(kv_lens, q, kc, vc, w.scale)
    O, L = decode_f64(q, kc, vc, kv_lens, w.scale)
    assert_close(o, lse, O, L, w.dtype, "decode workload")


@pytest.mark.parametrize("lens", [[1, 2, 3, 4], [255, 256, 257, 4096], [511, 512, 513, 1000],
                                  [4095, 4096, 1, 64], [0, 5, 0, 4096]])
def test_lengths_at_split_edges(lens):
    """kv_len = 0 (O = 0, LSE = -inf), 1, split boundaries +-1 and the full cache."""
    check(4, 32, 8, 4096, 128, "bf16", lens, seed=sum(lens))


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 4), (16, 2), (24, 8), (10, 2), (32, 2)])
@pytest.mark.parametrize("d,dtype", [(64, "fp16"), (128, "bf16"), (128, "fp16")])
def test_groupings_and_dims(Hq, Hkv, d, dtype):
    """G = Hq/Hkv in {1, 2, 3, 5, 8, 16}; G > 8 and odd G use head tiles with masking."""
    check(3, Hq, Hkv, 700, d, dtype, [700, 333, 1], seed=Hq + Hkv + d)


@pytest.mark.parametrize("d,dtype", [(64, "fp16"), (128, "bf16"), (128, "fp16")])
def test_growing_scores_force_rescales(d, dtype):
    """Scores that grow along the cache by about 10 (log2 units) per 64 tokens: every tile
    of every split raises the running maximum past the lazy-rescale threshold."""
    B, Hq, Hkv, cache = 4, 8, 2, 4096
    lens = [700, 2047, 3000, 4096]
    kv_lens, q, kc, vc = make_decode_inputs(B, Hq, Hkv, cache, d, dtype, 1, cache, seed=d,
                                            kv_lens=torch.tensor(lens))
    scale = 1.0 / math.sqrt(d)
    alpha = 10.0 / 64.0 / (scale * math.log2(math.e))
    q[..., 0] = 1.0
    kc[..., 0] = (torch.arange(cache, dtype=torch.float64) * alpha).to(kc.dtype)
    o, lse = run_decode(kv_lens, q, kc, vc, scale)
    O, L = decode_f64(q, kc, vc, kv_lens, scale)
    assert_close(o, lse, O, L, dtype, f"decode growing scores d{d} {dtype}", strict=False)


def test_poisoned_cache_rows_beyond_length():
    """NaN in cache rows >= kv_len must never be read."""
    B, Hq, Hkv, cache, d = 4, 16, 4, 2048, 128
    lens = torch.tensor([100, 2047, 1, 1500])
    kv_lens, q, kc, vc = make_decode_inputs(B, Hq, Hkv, cache, d, "bf16", 1, cache, 21,
                                            kv_lens=lens)
    kcp, vcp = kc.clone(), vc.clone()
    for b in range(B):
        kcp[b, :, int(lens[b]):] = float("nan")
        vcp[b, :, int(lens[b]):] = float("nan")
    o, lse = run_decode(kv_lens, q, kcp, vcp, 1 / math.sqrt(d))
    O, L = decode_f64(q, kc, vc, kv_lens, 1 / math.sqrt(d))
    assert_close(o, lse, O, L, "bf16", "poisoned decode", strict=False)


def test_lengths_beyond_cache_are_clamped():
    B, Hq, Hkv, cache, d = 2, 8, 2, 300, 64
    kv_lens, q, kc, vc = make_decode_inputs(B, Hq, Hkv, cache, d, "fp16", 1, cache, 22,
                                            kv_lens=torch.tensor([5000, -3]))
    o, lse = run_decode(kv_lens, q, kc, vc, 0.125)
    O, L = decode_f64(q, kc, vc, torch.tensor([300, 0]), 0.125)
    assert_close(o, lse, O, L, "fp16", "clamped", strict=False)


def test_workspace_reuse_and_determinism():
    w = WORKLOADS["decode"]
    kv_lens, q, kc, vc = make_decode_inputs(8, w.Hq, w.Hkv, 1024, w.d, w.dtype, 1, 1024, 23)
    ws = torch.empty(fa.decode_workspace_bytes(8, w.Hq, 1024, w.d), dtype=torch.uint8, device=DEV)
    ws.fill_(0xFF)   # garbage (NaN patterns) in the workspace must not matter
    args = (q.to(DEV), kc.to(DEV), vc.to(DEV), kv_lens.to(DEV))
    o1, l1 = fa.decode(*args, workspace=ws)
    o2, l2 = fa.decode(*args, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    O, L = decode_f64(q, kc, vc, kv_lens, w.scale)
    assert_close(o1.cpu(), l1.cpu(), O, L, w.dtype, "reuse", strict=False)


def test_many_sequences_every_tail_size():
    """160 sequences on the d = 128 tensor-core path (562 work units over the 148
    persistent CTAs) with lengths that give every ragged last-split size (1 to 8 tiles of
    128 tokens), exact multiples of the 1024-token split, single splits, empty, negative
    and over-capacity lengths, in a seeded shuffle. Outputs start as NaN, so a unit or a
    merge that is skipped shows."""
    B, Hq, Hkv, cache, d = 160, 8, 2, 2304, 128
    edge = [0, 1, 127, 128, 129, 255, 640, 1000, 1023, 1024, 1025, 1151, 1152, 1153, 1500,
            2047, 2048, 2049, 2175, 2176, 2303, 2304, -5, 9999]
    gen = torch.Generator().manual_seed(5)
    rand = torch.randint(0, cache + 1, (B - len(edge),), generator=gen).tolist()
    lens = edge + rand
    lens = [lens[i] for i in torch.randperm(B, generator=gen).tolist()]
    kv_lens, q, kc, vc = make_decode_inputs(B, Hq, Hkv, cache, d, "bf16", 1, cache, 6,
                                            kv_lens=torch.tensor(lens))
    scale = 1.0 / math.sqrt(d)
    o = torch.full((B, Hq, d), float("nan"), dtype=q.dtype, device=DEV)
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=DEV)
    fa.decode(q.to(DEV), kc.to(DEV), vc.to(DEV), kv_lens.to(DEV), scale=scale, out=o, lse=lse)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    clamped = torch.tensor([min(max(n, 0), cache) for n in lens])
    O, L = decode_f64(q, kc, vc, clamped, scale)
    assert_close(o.cpu(), lse.cpu(), O, L, "bf16", "every tail size", strict=False)


def test_bounded_wait_reports_timeout_and_context_survives():
    """Test hook: the d = 128 decode never loads its query rows, so every wait on them runs
    out after 20 ms; the split kernel records FA_ERR_DEVICE_TIMEOUT, drains and returns, and
    the next call (whose counter reset zeroes the ticket counter left behind) is correct."""
    lens = [700, 1500, 33, 4096]
    kv_lens, q, kc, vc = make_decode_inputs(4, 8, 2, 4096, 128, "bf16", 1, 4096, 5,
                                            kv_lens=torch.tensor(lens))
    qd, kd, vd, ld = q.to(DEV), kc.to(DEV), vc.to(DEV), kv_lens.to(DEV)
    scale = 1.0 / math.sqrt(128)
    torch.cuda.synchronize()
    assert fa.device_status(clear=True) == fa.FA_OK
    fa.set_wait_timeout_ns(20_000_000)
    fa.debug_skip_q_load(True)
    try:
        fa.decode(qd, kd, vd, ld, scale=scale)
        torch.cuda.synchronize()
        status = fa.device_status(clear=True)
    finally:
        fa.debug_skip_q_load(False)
        fa.set_wait_timeout_ns(0)
    assert status == fa.FA_ERR_DEVICE_TIMEOUT
    check(4, 8, 2, 4096, 128, "bf16", lens, seed=5)


def test_bounded_wait_reports_timeout_and_context_survives_cuda_cores():
    """Test hook on the CUDA-core decode (d = 64): the K/V ring stages are armed but never
    filled, so every wait on them runs out after 20 ms; the kernel records
    FA_ERR_DEVICE_TIMEOUT, drains and returns, and the next call is correct."""
    lens = [300, 64, 1000, 5]
    kv_lens, q, kc, vc = make_decode_inputs(4, 8, 4, 1024, 64, "fp16", 1, 1024, 6,
                                            kv_lens=torch.tensor(lens))
    qd, kd, vd, ld = q.to(DEV), kc.to(DEV), vc.to(DEV), kv_lens.to(DEV)
    torch.cuda.synchronize()
    assert fa.device_status(clear=True) == fa.FA_OK
    fa.set_wait_timeout_ns(20_000_000)
    fa.debug_skip_q_load(True)
    try:
        fa.decode(qd, kd, vd, ld, scale=0.125)
        torch.cuda.synchronize()
        status = fa.device_status(clear=True)
    finally:
        fa.debug_skip_q_load(False)
        fa.set_wait_timeout_ns(0)
    assert status == fa.FA_ERR_DEVICE_TIMEOUT
    check(4, 8, 4, 1024, 64, "fp16", lens, seed=6)
