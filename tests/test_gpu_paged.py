"""GPU parity of the paged-KV-cache entry points (fa_decode_paged, fa_fwd_paged) with the
float64 paged oracle. Pools are laid out by seeded random page tables (consecutive tokens
land in scattered pages); every pool row that holds no token of a sequence is NaN, so a
kernel that reads one shows it."""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_28_b200 as fa
from oracle.paged import attention_paged_rows_f64, decode_paged_f64
from tests.parity import assert_close, sample_rows
from workloads import WORKLOADS, make_decode_inputs, make_fwd_inputs, make_page_table, paginate

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def paged_decode_case(B, Hq, Hkv, ps, max_pages, d, dtype, lens, seed):
    cache = max_pages * ps
    kv_lens, q, kc, vc = make_decode_inputs(B, Hq, Hkv, cache, d, dtype, 1, cache, seed,
                                            kv_lens=torch.tensor(lens))
    table, P = make_page_table(kv_lens, ps, max_pages, seed=seed)
    kp = paginate(kc, table, kv_lens, ps, P)
    vp = paginate(vc, table, kv_lens, ps, P)
    return kv_lens, q, kp, vp, table


def run_decode_paged(kv_lens, q, kp, vp, table, scale, expect=fa.FA_OK):
    o, lse = fa.decode_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), table.to(DEV), kv_lens.to(DEV),
                             scale=scale)
    torch.cuda.synchronize()
    assert fa.device_status() == expect
    return o.cpu(), lse.cpu()


def check_decode(B, Hq, Hkv, ps, max_pages, d, dtype, lens, seed=0, strict=False):
    kv_lens, q, kp, vp, table = paged_decode_case(B, Hq, Hkv, ps, max_pages, d, dtype, lens, seed)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_decode_paged(kv_lens, q, kp, vp, table, scale)
    O, L = decode_paged_f64(q, kp, vp, table, kv_lens, ps, scale)
    return assert_close(o, lse, O, L, dtype,
                        f"paged decode ps{ps} B{B} Hq{Hq} Hkv{Hkv} d{d} {dtype} {lens}",
                        strict=strict)


@pytest.mark.parametrize("ps", [16, 256])
def test_decode_workload_paged_full(ps):
    """The 64-sequence GQA decode workload (Hq 32, Hkv 8, d 128, bf16, kv_len ~ U[512,4096],
    seed 0) with its cache in pages: every output."""
    w = WORKLOADS["decode"]
    kv_lens, _, _, _ = make_decode_inputs(w.B, w.Hq, w.Hkv, 1, w.d, w.dtype, w.kv_len_lo,
                                          w.kv_len_hi, w.seed)
    check_decode(w.B, w.Hq, w.Hkv, ps, w.N // ps, w.d, w.dtype, kv_lens.tolist(), seed=w.seed,
                 strict=True)


@pytest.mark.parametrize("d,dtype", [(64, "fp16"), (128, "bf16")])
@pytest.mark.parametrize("ps", [16, 32, 64, 128, 256, 1024])
def test_decode_page_sizes(ps, d, dtype):
    """Lengths at page and tile edges: 0 (O = 0, LSE = -inf), 1, ps - 1, ps, ps + 1, a long
    ragged one and the whole table."""
    max_pages = max(4, 2048 // ps)
    full = max_pages * ps
    lens = [0, 1, ps - 1, ps, ps + 1, 1000, full]
    check_decode(len(lens), 16, 4, ps, max_pages, d, dtype, lens, seed=ps + d)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 2), (10, 2), (32, 2)])
@pytest.mark.parametrize("d,dtype", [(64, "fp16"), (128, "bf16")])
def test_decode_paged_groupings(Hq, Hkv, d, dtype):
    check_decode(3, Hq, Hkv, 32, 24, d, dtype, [700, 333, 1], seed=Hq + Hkv + d)


@pytest.mark.parametrize("d,dtype", [(64, "fp16"), (128, "bf16")])
def test_decode_table_entry_outside_pool_is_reported(d, dtype):
    """An entry past the pool (or negative) is never dereferenced: the status word says
    FA_ERR_INVALID_ARG and the other sequences are unaffected."""
    lens = [300, 200, 150]
    kv_lens, q, kp, vp, table = paged_decode_case(3, 8, 2, 64, 8, d, dtype, lens, seed=31)
    bad = table.clone()
    bad[1, 1] = kp.shape[0] + 5
    bad[2, 0] = -7
    scale = 1.0 / math.sqrt(d)
    o, lse = run_decode_paged(kv_lens, q, kp, vp, bad, scale, expect=fa.FA_ERR_INVALID_ARG)
    assert fa.device_status() == fa.FA_OK          # cleared by the previous read
    O, L = decode_paged_f64(q, kp, vp, table, kv_lens, 64, scale)
    assert_close(o[:1], lse[:1], O[:1], L[:1], dtype, "unaffected sequence", strict=False)


def oracle_fwd_paged(q, kp, vp, table, Nk, ps, causal, scale):
    B, Hq, Nq, d = q.shape
    O = np.zeros((B, Hq, Nq, d))
    L = np.zeros((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            O[b, h], L[b, h] = attention_paged_rows_f64(q, kp, vp, table, Nk, ps, causal, scale, b,
                                                        h, np.arange(Nq))
    return O, L


def paged_fwd_case(B, Hq, Hkv, Nq, Nk, d, dtype, ps, seed, spare_pages=3):
    q, k, v = make_fwd_inputs(B, Hq, Hkv, Nq, Nk, d, dtype, seed=seed)
    max_pages = (Nk + ps - 1) // ps + 1
    lens = torch.full((B,), Nk)
    table, P = make_page_table(lens, ps, max_pages, spare_pages=spare_pages, seed=seed)
    return q, paginate(k, table, lens, ps, P), paginate(v, table, lens, ps, P), table


@pytest.mark.parametrize("d,dtype", [(64, "fp16"), (128, "bf16")])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("ps", [16, 64, 256])
@pytest.mark.parametrize("Nq,Nk", [(64, 300), (512, 1536), (1, 777), (256, 256), (300, 129)])
def test_prefill_paged(d, dtype, causal, ps, Nq, Nk):
    """A chunk of Nq queries against Nk paged tokens (bottom-right causal); the last page's
    rows past Nk and all unused pages are NaN."""
    B, Hq, Hkv = 2, 4, 2
    q, kp, vp, table = paged_fwd_case(B, Hq, Hkv, Nq, Nk, d, dtype, ps, seed=Nq + 7 * Nk + ps)
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.fwd_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), table.to(DEV), Nk, causal=causal,
                          scale=scale)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    O, L = oracle_fwd_paged(q, kp, vp, table, Nk, ps, causal, scale)
    assert_close(o.cpu(), lse.cpu(), O, L, dtype,
                 f"paged prefill d{d} {dtype} c{causal} ps{ps} Nq{Nq} Nk{Nk}", strict=False)


@pytest.mark.parametrize("d,dtype", [(64, "fp16"), (128, "bf16")])
def test_prefill_paged_table_entry_outside_pool_is_reported(d, dtype):
    q, kp, vp, table = paged_fwd_case(2, 4, 2, 128, 600, d, dtype, 64, seed=41)
    bad = table.clone()
    bad[1, 3] = 1 << 30
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.fwd_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), bad.to(DEV), 600, causal=True,
                          scale=scale)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_ERR_INVALID_ARG
    O, L = oracle_fwd_paged(q[:1], kp, vp, table[:1], 600, 64, True, scale)
    assert_close(o[:1].cpu(), lse[:1].cpu(), O, L, dtype, "unaffected sequence", strict=False)


@pytest.mark.parametrize("ps", [16, 128])
def test_gqa8k_paged_sampled_rows(ps):
    """Causal GQA prefill at full size (Hq 32, Hkv 8, 8192 tokens, d 128, bf16) from a
    paged pool: tile-edge and random rows of four heads."""
    w = WORKLOADS["gqa8k"]
    q, kp, vp, table = paged_fwd_case(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, ps, seed=w.seed)
    o, lse = fa.fwd_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), table.to(DEV), w.N, causal=True,
                          scale=w.scale)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    o, lse = o.cpu(), lse.cpu()
    rows = sample_rows(w.N, 48, seed=ps)
    for h in (0, 3, 17, 31):
        O, L = attention_paged_rows_f64(q, kp, vp, table, w.N, ps, True, w.scale, 0, h, rows)
        assert_close(o[0, h, rows], lse[0, h, rows], O, L, w.dtype, f"gqa8k paged ps{ps} h{h}")
