"""GPU parity of per-sequence lengths (q_lens, kv_lens) in fa_fwd_kvcache and fa_fwd_paged
with the float64 per-sequence oracles. Query rows past q_lens[b], cache rows past
kv_lens[b], pool rows that hold no token of a sequence and block-table entries past a
sequence's pages are all NaN or -1, so a kernel that reads them shows it; output rows past
q_lens[b] must keep the values the caller left there."""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_28_b200 as fa
from oracle import attention_paged_varlen_f64, attention_rows_f64, attention_varlen_f64
from tests.parity import assert_close, sample_rows, to_f64
from workloads import make_fwd_inputs, make_page_table, paginate

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
O_FILL, L_FILL = 7.0, 9.0


def poisoned_inputs(B, Hq, Hkv, Nq, cache, d, dtype, ql, kl, seed):
    q, kc, vc = make_fwd_inputs(B, Hq, Hkv, Nq, cache, d, dtype, seed)
    for b in range(B):
        q[b, :, max(ql[b], 0):] = float("nan")
        kc[b, :, max(kl[b], 0):] = float("nan")
        vc[b, :, max(kl[b], 0):] = float("nan")
    return q, kc, vc


def outputs(q):
    o = torch.full(q.shape, O_FILL, dtype=q.dtype, device=DEV)
    lse = torch.full(q.shape[:3], L_FILL, dtype=torch.float32, device=DEV)
    return o, lse


def check(o, lse, O, L, ql, dtype, what):
    """Rows below q_lens[b] against the oracle; rows at or past it untouched."""
    o, lse = o.cpu(), lse.cpu()
    B, Hq, Nq, _ = o.shape
    got_o, got_l, ref_o, ref_l = [], [], [], []
    for b in range(B):
        n = min(max(ql[b], 0), Nq)
        assert torch.all(o[b, :, n:] == O_FILL) and torch.all(lse[b, :, n:] == L_FILL), \
            f"{what}: rows past q_lens[{b}] = {n} were written"
        if n:
            got_o.append(to_f64(o[b, :, :n]).reshape(-1, o.shape[-1]))
            got_l.append(to_f64(lse[b, :, :n]).reshape(-1))
            ref_o.append(O[b, :, :n].reshape(-1, o.shape[-1]))
            ref_l.append(L[b, :, :n].reshape(-1))
    return assert_close(np.concatenate(got_o), np.concatenate(got_l), np.concatenate(ref_o),
                        np.concatenate(ref_l), dtype, what, strict=False)


# (nq_b, nk_b): empty query set, one token, full capacity, more queries than keys (causal
# rows that see nothing), no keys at all, a chunk against a longer prefix.
QL = [0, 1, 300, 77, 200, 129]
KL = [50, 1, 700, 64, 0, 513]


@pytest.mark.parametrize("d,dtype", [(64, "fp16"), (128, "bf16"), (64, "bf16"), (128, "fp16")])
@pytest.mark.parametrize("causal", [False, True])
def test_kvcache_per_sequence_lengths(d, dtype, causal):
    B, Hq, Hkv, Nq, Nk, cache = 6, 4, 2, 300, 700, 768
    q, kc, vc = poisoned_inputs(B, Hq, Hkv, Nq, cache, d, dtype, QL, KL, seed=d + causal)
    scale = 1.0 / math.sqrt(d)
    o, lse = outputs(q)
    fa.fwd_kvcache(q.to(DEV), kc.to(DEV), vc.to(DEV), Nk, causal=causal, scale=scale, out=o, lse=lse,
                   q_lens=torch.tensor(QL, dtype=torch.int32, device=DEV),
                   kv_lens=torch.tensor(KL, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    O, L = attention_varlen_f64(q, kc, vc, QL, KL, causal, scale)
    check(o, lse, O, L, QL, dtype, f"kvcache varlen d{d} {dtype} c{causal}")


def test_kvcache_one_length_array_only():
    """q_lens alone (every sequence has Nk keys) and kv_lens alone (Nq query rows each)."""
    B, Hq, Hkv, Nq, Nk, d = 3, 4, 1, 200, 400, 128
    scale = 1.0 / math.sqrt(d)
    for which, ql, kl in (("q_lens", [200, 5, 131], [Nk] * 3), ("kv_lens", [Nq] * 3, [400, 130, 199])):
        q, kc, vc = poisoned_inputs(B, Hq, Hkv, Nq, Nk, d, "bf16", ql, kl, seed=ql[1] + kl[1])
        o, lse = outputs(q)
        lens = torch.tensor(ql if which == "q_lens" else kl, dtype=torch.int32, device=DEV)
        fa.fwd_kvcache(q.to(DEV), kc.to(DEV), vc.to(DEV), Nk, causal=True, scale=scale, out=o, lse=lse,
                       **{which: lens})
        torch.cuda.synchronize()
        assert fa.device_status() == fa.FA_OK
        O, L = attention_varlen_f64(q, kc, vc, ql, kl, True, scale)
        check(o, lse, O, L, ql, "bf16", f"{which} only")


def test_lengths_out_of_range_are_clamped():
    """Negative lengths act as 0, lengths past the capacity as the capacity."""
    B, Hq, Hkv, Nq, Nk, d = 4, 2, 2, 130, 260, 64
    ql, kl = [-5, 500, 64, 130], [100, 999, -1, 260]
    qc, kcl = [0, 130, 64, 130], [100, 260, 0, 260]
    q, kc, vc = poisoned_inputs(B, Hq, Hkv, Nq, Nk, d, "fp16", qc, kcl, seed=21)
    o, lse = outputs(q)
    fa.fwd_kvcache(q.to(DEV), kc.to(DEV), vc.to(DEV), Nk, causal=True, scale=0.125, out=o, lse=lse,
                   q_lens=torch.tensor(ql, dtype=torch.int32, device=DEV),
                   kv_lens=torch.tensor(kl, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    O, L = attention_varlen_f64(q, kc, vc, qc, kcl, True, 0.125)
    check(o, lse, O, L, qc, "fp16", "clamped lengths")


@pytest.mark.parametrize("ps", [16, 64, 256])
@pytest.mark.parametrize("d,dtype", [(64, "fp16"), (128, "bf16")])
@pytest.mark.parametrize("causal", [False, True])
def test_paged_per_sequence_lengths(ps, d, dtype, causal):
    """Key counts at page edges (minus one, exact, plus one) and at key-tile edges; pages
    scattered by a seeded table, every unused pool row NaN, unused table entries -1."""
    kl = [ps - 1, ps, ps + 1, 2 * ps + 1, 3 * ps - 1, 5, 128, 129]
    ql = [min(x, y) for x, y in zip(kl, [ps, 7, ps + 1, 40, 3 * ps - 1, 5, 128, 200])]
    ql[-1] = 200                                        # more queries than keys
    B, Hq, Hkv, d_ = len(kl), 4, 2, d
    cap = max(kl)
    max_pages = (cap + ps - 1) // ps
    Nq = max(ql)
    q, kc, vc = poisoned_inputs(B, Hq, Hkv, Nq, max_pages * ps, d_, dtype, ql, kl, seed=ps + d)
    lens = torch.tensor(kl)
    table, P = make_page_table(lens, ps, max_pages, seed=ps + d)
    kp, vp = paginate(kc, table, lens, ps, P), paginate(vc, table, lens, ps, P)
    scale = 1.0 / math.sqrt(d)
    o, lse = outputs(q)
    fa.fwd_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), table.to(DEV), cap, causal=causal, scale=scale,
                 out=o, lse=lse, q_lens=torch.tensor(ql, dtype=torch.int32, device=DEV),
                 kv_lens=torch.tensor(kl, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    O, L = attention_paged_varlen_f64(q, kp, vp, table, ql, kl, ps, causal, scale)
    check(o, lse, O, L, ql, dtype, f"paged varlen ps{ps} d{d} {dtype} c{causal}")


def test_two_chunks_per_sequence_equal_whole_sequences():
    """A ragged batch prefilled in two calls (each sequence's first chunk, then the rest
    against the whole prefix) gives every sequence's full causal attention."""
    B, Hq, Hkv, d, cap = 4, 8, 2, 128, 1024
    total = [1024, 600, 257, 33]
    first = [512, 100, 256, 0]
    q, kc, vc = make_fwd_inputs(B, Hq, Hkv, cap, cap, d, "bf16", seed=31)
    scale = 1.0 / math.sqrt(d)
    qd, kd, vd = q.to(DEV), kc.to(DEV), vc.to(DEV)
    o_full = torch.full(q.shape, O_FILL, dtype=q.dtype, device=DEV)
    l_full = torch.full(q.shape[:3], L_FILL, dtype=torch.float32, device=DEV)
    # chunk 1: rows [0, first) against keys [0, first)
    fa.fwd_kvcache(qd, kd, vd, cap, causal=True, scale=scale, out=o_full, lse=l_full,
                   q_lens=torch.tensor(first, dtype=torch.int32, device=DEV),
                   kv_lens=torch.tensor(first, dtype=torch.int32, device=DEV))
    # chunk 2: rows [first, total), packed at the start of their own buffer
    n2 = [t - f for t, f in zip(total, first)]
    q2 = torch.zeros((B, Hq, max(n2), d), dtype=q.dtype)
    for b in range(B):
        q2[b, :, :n2[b]] = q[b, :, first[b]:total[b]]
    o2 = torch.full(q2.shape, O_FILL, dtype=q.dtype, device=DEV)
    l2 = torch.full(q2.shape[:3], L_FILL, dtype=torch.float32, device=DEV)
    fa.fwd_kvcache(q2.to(DEV), kd, vd, cap, causal=True, scale=scale, out=o2, lse=l2,
                   q_lens=torch.tensor(n2, dtype=torch.int32, device=DEV),
                   kv_lens=torch.tensor(total, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    o_full, l_full, o2, l2 = o_full.cpu(), l_full.cpu(), o2.cpu(), l2.cpu()
    for b in range(B):
        o_full[b, :, first[b]:total[b]] = o2[b, :, :n2[b]]
        l_full[b, :, first[b]:total[b]] = l2[b, :, :n2[b]]
    O, L = attention_varlen_f64(q, kc, vc, total, total, True, scale)
    check(o_full.to(DEV), l_full.to(DEV), O, L, total, "bf16", "two chunks")


def test_ragged_gqa8k_batch_sampled_rows():
    """A ragged batch of the 8B-class layer shape (Hq 32, Hkv 8, d 128, bf16, cache 8192):
    a full 8192-token prefill, a 1000-token chunk after a 4000-token prefix, a 2049-token
    prefill and one decode-like row; seeded rows of every head against the oracle."""
    B, Hq, Hkv, d, cap = 4, 32, 8, 128, 8192
    kl, ql = [8192, 5000, 2049, 700], [8192, 1000, 2049, 1]
    q, kc, vc = poisoned_inputs(B, Hq, Hkv, cap, cap, d, "bf16", ql, kl, seed=41)
    scale = 1.0 / math.sqrt(d)
    o, lse = outputs(q)
    fa.fwd_kvcache(q.to(DEV), kc.to(DEV), vc.to(DEV), cap, causal=True, scale=scale, out=o, lse=lse,
                   q_lens=torch.tensor(ql, dtype=torch.int32, device=DEV),
                   kv_lens=torch.tensor(kl, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    o, lse = o.cpu(), lse.cpu()
    for b in range(B):
        assert torch.all(o[b, :, ql[b]:] == O_FILL) and torch.all(lse[b, :, ql[b]:] == L_FILL)
        rows = sample_rows(ql[b], 24, seed=b)
        qb, kb, vb = q[b:b + 1, :, :ql[b]], kc[b:b + 1, :, :kl[b]], vc[b:b + 1, :, :kl[b]]
        for h in range(Hq):
            O, L = attention_rows_f64(qb, kb, vb, True, scale, 0, h, rows)
            assert_close(o[b, h, rows], lse[b, h, rows], O, L, "bf16", f"ragged b{b} h{h}", strict=False)


def test_many_units_with_empty_sequences_interleaved():
    """More work units than resident CTAs at d = 64 (two CTAs per SM, so CTAs take over
    units that have not started), with sequences that have no queries or no keys among
    full ones: consecutive units of one CTA alternate between units with key tiles and
    units without any."""
    B, Hq, Hkv, N, d = 48, 12, 12, 512, 64
    ql = [0 if b % 3 == 1 else N for b in range(B)]
    kl = [0 if b % 3 == 2 else N for b in range(B)]
    q, kc, vc = poisoned_inputs(B, Hq, Hkv, N, N, d, "fp16", ql, kl, seed=51)
    o, lse = outputs(q)
    fa.fwd_kvcache(q.to(DEV), kc.to(DEV), vc.to(DEV), N, causal=True, scale=0.125, out=o, lse=lse,
                   q_lens=torch.tensor(ql, dtype=torch.int32, device=DEV),
                   kv_lens=torch.tensor(kl, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    o, lse = o.cpu(), lse.cpu()
    rows = sample_rows(N, 16, seed=5)
    for b in range(B):
        if ql[b] == 0:
            assert torch.all(o[b] == O_FILL) and torch.all(lse[b] == L_FILL)
        elif kl[b] == 0:
            assert torch.all(o[b] == 0) and torch.all(torch.isneginf(lse[b]))
        elif b % 6 == 0:
            for h in (0, Hq - 1):
                O, L = attention_rows_f64(q[b:b + 1], kc[b:b + 1], vc[b:b + 1], True, 0.125, 0, h, rows)
                assert_close(o[b, h, rows], lse[b, h, rows], O, L, "fp16", f"interleaved b{b} h{h}",
                             strict=False)


def test_ragged_grouped_query_batch_of_four_sequences():
    """Per-sequence lengths in a grouped-query batch with 67 MB of K/V capacity (B=4,
    Hq=8, Hkv=4, cache 8192): a full sequence, a short one, one without keys and a chunk
    after a long prefix."""
    B, Hq, Hkv, cap, d = 4, 8, 4, 8192, 128
    kl, ql = [8192, 100, 0, 5000], [8192, 100, 7, 1000]
    q, kc, vc = poisoned_inputs(B, Hq, Hkv, cap, cap, d, "bf16", ql, kl, seed=71)
    scale = 1.0 / math.sqrt(d)
    o, lse = outputs(q)
    fa.fwd_kvcache(q.to(DEV), kc.to(DEV), vc.to(DEV), cap, causal=True, scale=scale, out=o, lse=lse,
                   q_lens=torch.tensor(ql, dtype=torch.int32, device=DEV),
                   kv_lens=torch.tensor(kl, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    o, lse = o.cpu(), lse.cpu()
    for b in range(B):
        assert torch.all(o[b, :, ql[b]:] == O_FILL) and torch.all(lse[b, :, ql[b]:] == L_FILL)
        if kl[b] == 0:
            assert torch.all(o[b, :, :ql[b]] == 0) and torch.all(torch.isneginf(lse[b, :, :ql[b]]))
            continue
        rows = sample_rows(ql[b], 16, seed=b)
        qb, kb, vb = q[b:b + 1, :, :ql[b]], kc[b:b + 1, :, :kl[b]], vc[b:b + 1, :, :kl[b]]
        for h in (0, Hq - 1):
            O, L = attention_rows_f64(qb, kb, vb, True, scale, 0, h, rows)
            assert_close(o[b, h, rows], lse[b, h, rows], O, L, "bf16", f"ragged gqa b{b} h{h}",
                         strict=False)
