"""fa_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc where they decode: a serving process that has given
nearly all device memory to its own pool and KV cache, a plugin handed tensors but no
allocator, or a latency-critical loop that must avoid cudaMalloc's cost and implicit
synchronisation. fa_decode_noalloc serves them with the library's own fixed scratch array.
These tests check it through the C ABI against fa_decode with a caller workspace, on two
calls in a row (the second sees the first call's leftovers in the shared scratch).

This file is named so that pytest collects it last.
"""
import math

import pytest
import torch

import io_aware_exact_28_b200 as fa
from tests.parity import MAX_ABS, RMS_TOL, metrics, to_f64
from workloads import WORKLOADS, make_decode_inputs

DEV = "cuda:0"


def test_oversized_request_is_rejected_before_any_launch():
    """Sizes whose scratch would exceed the fixed 32 MiB are refused on the host."""
    need = fa.decode_workspace_bytes(256, 64, 65536, 128)
    assert need > fa.DECODE_NOALLOC_SCRATCH_BYTES
    st = fa.lib().fa_decode_noalloc(16, 16, 16, 16, 16, None, 256, 64, 8, 65536, 128, 0.088, 1, None)
    assert st == fa.FA_ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_decode_on_two_calls_in_a_row():
    w = WORKLOADS["decode"]
    scale = 1.0 / math.sqrt(w.d)
    cases = [
        make_decode_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.dtype, w.kv_len_lo, w.kv_len_hi, w.seed),
        make_decode_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.dtype, 1, w.N, seed=7),
    ]
    assert fa.decode_workspace_bytes(w.B, w.Hq, w.N, w.d) <= fa.DECODE_NOALLOC_SCRATCH_BYTES
    for i, (kv_lens, q, kc, vc) in enumerate(cases):
        args = (q.to(DEV), kc.to(DEV), vc.to(DEV), kv_lens.to(DEV))
        o_ref, l_ref = fa.decode(*args, scale=scale)
        o_na, l_na = fa.decode_noalloc(*args, scale=scale)
        torch.cuda.synchronize()
        assert fa.device_status() == fa.FA_OK
        m = metrics(o_na.cpu(), l_na.cpu(), to_f64(o_ref.cpu()), to_f64(l_ref.cpu()))
        assert m["max_abs"] <= MAX_ABS[w.dtype], (i, m)
        assert m["rms"] <= RMS_TOL, (i, m)
        assert m["lse_nonfinite_mismatch"] == 0 and m["lse_rel"] <= 1e-4, (i, m)
        # same kernels, same split: the two paths agree bit for bit
        assert torch.equal(o_na, o_ref) and torch.equal(l_na, l_ref), i
