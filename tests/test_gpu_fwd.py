"""GPU parity of fa_fwd (through the C ABI) against the float64 CPU oracle."""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_28_b200 as fa
from oracle import attention_f64, attention_rows_f64
from tests.parity import LSE_REL, MAX_ABS, RMS_TOL, assert_close, sample_rows, to_f64
from workloads import WORKLOADS, make_fwd_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def run_fwd(q, k, v, causal, scale=None):
    o, lse = fa.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    return o.cpu(), lse.cpu()


def check_full(B, Hq, Hkv, Nq, Nk, d, dtype, causal, seed=0, strict=False):
    q, k, v = make_fwd_inputs(B, Hq, Hkv, Nq, Nk, d, dtype, seed)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_fwd(q, k, v, causal, scale)
    O, L = attention_f64(q, k, v, causal, scale)
    return assert_close(o, lse, O, L, dtype, f"B{B} Hq{Hq} Hkv{Hkv} Nq{Nq} Nk{Nk} d{d} {dtype} c{causal}",
                        strict=strict)


def test_tiny_workload():
    w = WORKLOADS["tiny"]
    check_full(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, w.causal, strict=True)


def test_mha2k_workload_full():
    """The causal B=8 H=12 N=2048 d=64 fp16 workload, every output element."""
    w = WORKLOADS["mha2k"]
    check_full(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, w.causal, strict=True)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 77, 128, 129, 256, 300, 640])
def test_shapes_ragged(d, dtype, causal, N):
    """Lengths that are not multiples of the 128-row tile or the 256-row CTA block."""
    check_full(1, 2, 1, N, N, d, dtype, causal, seed=N + d)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
def test_growing_scores_force_rescales(d, dtype, causal):
    """Scores that grow along the key axis by about 10 (log2 units) per 64 keys: the row
    maximum exceeds the lazy-rescale threshold on nearly every key tile, so the rescale of
    O and l, and at d = 128 the recomputation of P against the new maximum, run on almost
    every tile instead of almost never."""
    B, Hq, Hkv, N = 1, 2, 1, 640
    q, k, v = make_fwd_inputs(B, Hq, Hkv, N, N, d, dtype, seed=d + N)
    scale = 1.0 / math.sqrt(d)
    alpha = 10.0 / 64.0 / (scale * math.log2(math.e))
    q[..., 0] = 1.0
    k[..., 0] = (torch.arange(N, dtype=torch.float64) * alpha).to(k.dtype)
    o, lse = run_fwd(q, k, v, causal, scale)
    O, L = attention_f64(q, k, v, causal, scale)
    assert_close(o, lse, O, L, dtype, f"growing scores d{d} {dtype} c{causal}", strict=False)


@pytest.mark.parametrize("Nq,Nk", [(128, 640), (77, 300), (300, 77), (1, 513), (256, 129),
                                   (512, 1024)])
@pytest.mark.parametrize("causal", [False, True])
def test_rectangular(Nq, Nk, causal):
    """Nq != Nk, bottom-right aligned causal mask (chunked prefill against a longer prefix,
    and the degenerate Nq > Nk case where early rows see no key)."""
    check_full(2, 4, 2, Nq, Nk, 128, "bf16", causal, seed=Nq * 7 + Nk)


@pytest.mark.parametrize("Nq,Nk", [(300, 77), (640, 200), (512, 1024), (200, 1000)])
@pytest.mark.parametrize("causal", [False, True])
def test_rectangular_d64(Nq, Nk, causal):
    """The d = 64 kernel (64-key tiles) on rectangular shapes, including causal CTAs whose
    first query tile sees no key while the second does."""
    check_full(2, 4, 2, Nq, Nk, 64, "fp16", causal, seed=Nq * 5 + Nk)


@pytest.mark.parametrize("Hq,Hkv", [(8, 1), (8, 2), (6, 3), (4, 4)])
def test_gqa_groupings(Hq, Hkv):
    check_full(2, Hq, Hkv, 384, 384, 64, "fp16", True, seed=Hq * 10 + Hkv)


def test_first_causal_row_is_exact():
    """Row 0 of a square causal problem sees only key 0: P = 1, l = 1, O = V[0] exactly."""
    q, k, v = make_fwd_inputs(1, 4, 4, 512, 512, 128, "bf16", seed=11)
    o, lse = run_fwd(q, k, v, True)
    assert torch.equal(o[:, :, 0], v[:, :, 0])
    s00 = (q[:, :, 0].double() * k[:, :, 0].double()).sum(-1) / math.sqrt(128)
    assert np.allclose(lse[:, :, 0].double().numpy(), s00.numpy(), rtol=0, atol=2e-5)


def test_constant_v_gives_constant_o():
    q, k, _ = make_fwd_inputs(1, 2, 2, 384, 384, 64, "fp16", seed=12)
    c = torch.randn(64, generator=torch.Generator().manual_seed(13)).half()
    v = c.expand(1, 2, 384, 64).contiguous()
    o, _ = run_fwd(q, k, v, True)
    assert (o.float() - c.float()).abs().max().item() <= 2e-3


def test_one_hot_scores_select_one_value_row():
    """q = c e1, k_j* = e1, other keys 0, c*scale = 200: every other weight is 2^-288 (0 in
    fp32), so O = V[j*] exactly."""
    N, d = 256, 64
    q = torch.zeros(1, 1, N, d, dtype=torch.bfloat16)
    q[..., 0] = 1600.0
    k = torch.zeros(1, 1, N, d, dtype=torch.bfloat16)
    k[0, 0, 173, 0] = 1.0
    v = torch.randn(1, 1, N, d, generator=torch.Generator().manual_seed(14)).bfloat16()
    o, lse = run_fwd(q, k, v, False, scale=0.125)
    assert torch.equal(o[0, 0], v[0, 0, 173].expand(N, d))
    assert np.allclose(lse.numpy(), 200.0, rtol=0, atol=1e-4)


def test_poisoned_padding_and_guard_bands():
    """NaN in the memory right after K, V and Q must not leak into O; memory right after
    O and LSE must stay untouched (the kernel writes only [0, Nq) rows)."""
    N, d, pad = 200, 128, 256
    q, k, v = make_fwd_inputs(1, 1, 1, N, N, d, "bf16", seed=15)
    bufs = []
    for t in (q, k, v):
        b = torch.full((N + pad, d), float("nan"), dtype=torch.bfloat16, device=DEV)
        b[:N] = t[0, 0].to(DEV)
        bufs.append(b)
    obuf = torch.full((N + pad, d), 7.0, dtype=torch.bfloat16, device=DEV)
    lbuf = torch.full((N + pad,), 9.0, dtype=torch.float32, device=DEV)
    qv, kv, vv = (b[:N].view(1, 1, N, d) for b in bufs)
    fa.fwd(qv, kv, vv, causal=True, out=obuf[:N].view(1, 1, N, d), lse=lbuf[:N].view(1, 1, N))
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    O, L = attention_f64(q, k, v, True, 1 / math.sqrt(d))
    assert_close(obuf[:N].view(1, 1, N, d).cpu(), lbuf[:N].view(1, 1, N).cpu(), O, L, "bf16", "poison",
                 strict=False)
    assert torch.all(obuf[N:] == 7.0) and torch.all(lbuf[N:] == 9.0)


def test_lse_may_be_null():
    q, k, v = make_fwd_inputs(1, 2, 2, 256, 256, 64, "fp16", seed=16)
    o, lse = fa.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, return_lse=False)
    torch.cuda.synchronize()
    assert lse is None
    O, _ = attention_f64(q, k, v, True, 0.125)
    assert_close(o.cpu(), None, O, None, "fp16", "no-lse", strict=False)


def test_repeated_calls_are_deterministic():
    q, k, v = make_fwd_inputs(1, 4, 2, 1000, 1000, 128, "bf16", seed=17)
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    o1, l1 = fa.fwd(q, k, v, causal=True)
    o2, l2 = fa.fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bounded_wait_reports_timeout_and_context_survives():
    """Test hook: the Q load is never issued, so the waits on it run out after 20 ms; the
    kernel records FA_ERR_DEVICE_TIMEOUT and returns, and the next call works."""
    q, k, v = make_fwd_inputs(1, 1, 1, 256, 256, 64, "fp16", seed=18)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    assert fa.device_status(clear=True) == fa.FA_OK
    fa.set_wait_timeout_ns(20_000_000)
    fa.debug_skip_q_load(True)
    try:
        fa.fwd(qd, kd, vd, causal=True)
        status = fa.device_status(clear=True)
    finally:
        fa.debug_skip_q_load(False)
        fa.set_wait_timeout_ns(0)
    assert status == fa.FA_ERR_DEVICE_TIMEOUT
    o, lse = fa.fwd(qd, kd, vd, causal=True)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    O, L = attention_f64(q, k, v, True, 0.125)
    assert_close(o.cpu(), lse.cpu(), O, L, "fp16", "after-timeout", strict=False)


class _Stats:
    """Running comparison statistics over many blocks of one output (max-abs, RMS over
    every element, LSE relative error, -inf pattern)."""

    def __init__(self):
        self.max_abs, self.sq, self.n, self.lse_rel, self.lse_bad = 0.0, 0.0, 0, 0.0, 0

    def add(self, o, lse, O, L):
        err = np.abs(o - O)
        self.max_abs = max(self.max_abs, float(err.max()))
        self.sq += float(np.sum(err ** 2))
        self.n += err.size
        fin = np.isfinite(L)
        self.lse_bad += int(np.sum(np.isfinite(lse) != fin))
        if fin.any():
            rel = np.abs(lse[fin] - L[fin]) / np.maximum(np.abs(L[fin]), 1.0)
            self.lse_rel = max(self.lse_rel, float(rel.max()))

    def check(self, dtype, what):
        rms = math.sqrt(self.sq / max(self.n, 1))
        m = {"max_abs": self.max_abs, "rms": rms, "lse_rel": self.lse_rel, "elements": self.n}
        assert self.lse_bad == 0, f"{what}: -inf pattern of LSE differs {m}"
        assert self.max_abs <= MAX_ABS[dtype], f"{what}: max-abs {m}"
        assert rms <= RMS_TOL, f"{what}: rms {m}"
        assert self.lse_rel <= LSE_REL, f"{what}: LSE rel {m}"
        return m


def test_gqa8k_workload_every_element():
    """GQA causal prefill B=1 Hq=32 Hkv=8 N=8192 d=128 bf16, in the launch the benchmark
    times: every output element and every LSE against the oracle. The oracle runs head by
    head in 1024-row blocks; a causal row block [r0, r1) depends only on the first r1
    positions of Q, K and V, so each block is the oracle on that prefix (a property of the
    causal definition, so no S wider than the visible keys is formed)."""
    from concurrent.futures import ThreadPoolExecutor
    w = WORKLOADS["gqa8k"]
    q, k, v = make_fwd_inputs(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, w.seed)
    o, lse = run_fwd(q, k, v, True, w.scale)
    o64, l64 = to_f64(o), to_f64(lse)
    blk = 1024

    def head(h):
        st = _Stats()
        for r0 in range(0, w.N, blk):
            r1 = min(r0 + blk, w.N)
            O, L = attention_rows_f64(q[:, :, :r1], k[:, :, :r1], v[:, :, :r1], True, w.scale,
                                      0, h, np.arange(r0, r1))
            st.add(o64[0, h, r0:r1], l64[0, h, r0:r1], O, L)
        return st

    with ThreadPoolExecutor(max_workers=8) as ex:
        parts = list(ex.map(head, range(w.Hq)))
    total = _Stats()
    for st in parts:
        total.max_abs = max(total.max_abs, st.max_abs)
        total.sq += st.sq
        total.n += st.n
        total.lse_rel = max(total.lse_rel, st.lse_rel)
        total.lse_bad += st.lse_bad
    m = total.check(w.dtype, "gqa8k every element")
    assert m["elements"] == w.B * w.Hq * w.N * w.d
    print("gqa8k every element:", m)


def rows_256(N: int, seed: int) -> np.ndarray:
    """256 distinct query rows of a length-N sequence: rows 0, 1, 127, 128 and N-1, the
    other tile edges of `sample_rows`, then seeded random rows."""
    must = np.array([0, 1, 127, 128, N - 1], dtype=np.int64)
    edges = sample_rows(N, 0, seed)
    rows = np.unique(np.concatenate([must, edges]))
    rng = np.random.default_rng(seed)
    while len(rows) < 256:
        rows = np.unique(np.concatenate([rows, rng.choice(N, size=256 - len(rows), replace=False)]))
    return rows


def test_gqa32k_workload_256_rows_per_head():
    """Long-context GQA causal prefill B=1 Hq=32 Hkv=8 N=32768 d=128 bf16, in the launch
    the benchmark times: 256 seeded query rows of every head (rows 0, 1, 127, 128 and N-1
    among them) against the oracle, every element of those rows; and at every row, the
    output is finite and, being a convex combination of V rows, within max |V|."""
    from concurrent.futures import ThreadPoolExecutor
    w = WORKLOADS["gqa32k"]
    q, k, v = make_fwd_inputs(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, w.seed)
    o, lse = run_fwd(q, k, v, True, w.scale)

    def head(h):
        rows = rows_256(w.N, seed=w.N + h)
        assert len(rows) == 256 and {0, 1, 127, 128, w.N - 1} <= set(rows.tolist())
        O, L = attention_rows_f64(q, k, v, True, w.scale, 0, h, rows)
        st = _Stats()
        st.add(to_f64(o[0, h, rows]), to_f64(lse[0, h, rows]), O, L)
        return st

    with ThreadPoolExecutor(max_workers=8) as ex:
        parts = list(ex.map(head, range(w.Hq)))
    total = _Stats()
    for st in parts:
        total.max_abs = max(total.max_abs, st.max_abs)
        total.sq += st.sq
        total.n += st.n
        total.lse_rel = max(total.lse_rel, st.lse_rel)
        total.lse_bad += st.lse_bad
    m = total.check(w.dtype, "gqa32k 256 rows per head")
    assert m["elements"] == w.Hq * 256 * w.d
    print("gqa32k 256 rows per head:", m)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    assert o.float().abs().max() <= v.float().abs().max() + 1e-2


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,dtype,causal", [
    (8, 12, 12, 1024, 1024, 64, "fp16", False),   # 384 units: every unit has equal tile counts
    (2, 32, 8, 2048, 2048, 128, "bf16", False),   # 512 units on 148 SMs
    (8, 12, 12, 1024, 512, 64, "fp16", True),     # early query rows see no key
    (2, 32, 8, 2048, 1024, 128, "bf16", True),
])
def test_more_units_than_resident_ctas(B, Hq, Hkv, Nq, Nk, d, dtype, causal):
    """More work units than resident CTAs, so running CTAs take over the rest (cluster launch
    control); sampled rows of the first and last head against the oracle."""
    q, k, v = make_fwd_inputs(B, Hq, Hkv, Nq, Nk, d, dtype, seed=Nq + Nk + d)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_fwd(q, k, v, causal, scale)
    rows = sample_rows(Nq, 24, seed=1)
    for (b, h) in [(0, 0), (B - 1, Hq - 1)]:
        O, L = attention_rows_f64(q, k, v, causal, scale, b, h, rows)
        assert_close(o[b, h, rows], lse[b, h, rows], O, L, dtype, f"takeover b{b} h{h}", strict=False)


def test_kv_head_major_order_with_several_sequences():
    """Grouped-query calls whose K and V exceed half of L2 number their work units KV
    head by KV head (B=4, Hq=8, Hkv=4, N=8192, d=128: 67 MB of K/V); seeded rows of heads
    spread over every sequence and KV group against the oracle."""
    B, Hq, Hkv, N, d = 4, 8, 4, 8192, 128
    q, k, v = make_fwd_inputs(B, Hq, Hkv, N, N, d, "bf16", seed=61)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_fwd(q, k, v, True, scale)
    rows = sample_rows(N, 24, seed=61)
    for b, h in ((0, 0), (0, 7), (1, 3), (2, 4), (3, 0), (3, 7)):
        O, L = attention_rows_f64(q, k, v, True, scale, b, h, rows)
        assert_close(o[b, h, rows], lse[b, h, rows], O, L, "bf16", f"kv-major b{b} h{h}", strict=False)
