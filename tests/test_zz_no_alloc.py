"""fa_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc where they decode: a serving process that has given
nearly all device memory to its own pool and KV cache, a plugin handed tensors but no
allocator, or a latency-critical loop that must avoid cudaMalloc's cost and implicit
synchronisation. fa_decode_noalloc serves them with the library's own fixed scratch array.
These tests check it through the C ABI against fa_decode with a fresh caller workspace, on
two calls in a row within each test: a large layout first, then a smaller one whose
partial rows and LSE slots sit where the first call left its own, so stale contents of the
shared scratch would show. Each test makes its own first call, so none depends on what
ran before it in the process (the file name only places it at the end of a run).
"""
import math

import pytest
import torch

import io_aware_exact_28_b200 as fa
from tests.parity import MAX_ABS, RMS_TOL, metrics, to_f64
from workloads import make_decode_inputs

DEV = "cuda:0"


def test_oversized_request_is_rejected_before_any_launch():
    """Sizes whose scratch would exceed the fixed 32 MiB are refused on the host."""
    need = fa.decode_workspace_bytes(256, 64, 65536, 128)
    assert need > fa.DECODE_NOALLOC_SCRATCH_BYTES
    st = fa.lib().fa_decode_noalloc(16, 16, 16, 16, 16, None, 256, 64, 8, 65536, 128, 0.088, 1, None)
    assert st == fa.FA_ERR_WORKSPACE


@pytest.mark.gpu
@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (64, "fp16")])
def test_noalloc_decode_matches_workspace_decode_on_two_calls_in_a_row(d, dtype):
    """d = 128 runs the tensor-core split kernel, d = 64 the CUDA-core one; both leave
    partial rows and LSE values in the shared scratch for the next call to overwrite."""
    scale = 1.0 / math.sqrt(d)
    # (B, Hq, Hkv, cache capacity, seed): the first layout spans most of the scratch.
    layouts = [(32, 64, 4, 8192, 3), (8, 16, 2, 1024, 4)]
    sizes = [fa.decode_workspace_bytes(B, Hq, cap, d) for B, Hq, _, cap, _ in layouts]
    assert all(n <= fa.DECODE_NOALLOC_SCRATCH_BYTES for n in sizes)
    assert sizes[0] > 4 * sizes[1]
    for i, (B, Hq, Hkv, cap, seed) in enumerate(layouts):
        kv_lens, q, kc, vc = make_decode_inputs(B, Hq, Hkv, cap, d, dtype, 0, cap, seed=seed)
        kv_lens[0], kv_lens[-1] = 0, cap            # an empty sequence and a full one
        args = (q.to(DEV), kc.to(DEV), vc.to(DEV), kv_lens.to(DEV))
        o_ref, l_ref = fa.decode(*args, scale=scale)   # fresh workspace from the binding
        o_na, l_na = fa.decode_noalloc(*args, scale=scale)
        torch.cuda.synchronize()
        assert fa.device_status() == fa.FA_OK
        m = metrics(o_na.cpu(), l_na.cpu(), to_f64(o_ref.cpu()), to_f64(l_ref.cpu()))
        assert m["max_abs"] <= MAX_ABS[dtype], (i, m)
        assert m["rms"] <= RMS_TOL, (i, m)
        assert m["lse_nonfinite_mismatch"] == 0 and m["lse_rel"] <= 1e-4, (i, m)
        # same kernels, same split: the two paths agree bit for bit
        assert torch.equal(o_na, o_ref) and torch.equal(l_na, l_ref), i
        del args, kc, vc
