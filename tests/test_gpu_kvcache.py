"""GPU parity of fa_fwd_kvcache (chunked prefill against a KV cache) with the float64
oracle: a chunk of queries against the first Nk rows of a cache whose capacity exceeds
Nk, with bottom-right causal alignment (page "Flash Attention ... IO-aware exact" (fr),
manual chunking example; "Optimisation avancée : KV Cache")."""
import math

import pytest
import torch

import io_aware_exact_28_b200 as fa
from oracle import attention_f64
from tests.parity import assert_close
from workloads import make_fwd_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def run(q, kc, vc, nk, causal, scale):
    o, lse = fa.fwd_kvcache(q.to(DEV), kc.to(DEV), vc.to(DEV), nk, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    return o.cpu(), lse.cpu()


@pytest.mark.parametrize("d,dtype", [(64, "fp16"), (128, "bf16")])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk,cache", [(64, 300, 512), (512, 1536, 4096), (1, 777, 1024),
                                         (256, 256, 300), (300, 129, 1000)])
def test_prefix_of_a_larger_cache(d, dtype, causal, Nq, Nk, cache):
    """Rows [Nk, cache) of the cache hold NaN: they must never reach the result."""
    B, Hq, Hkv = 2, 4, 2
    q, kc, vc = make_fwd_inputs(B, Hq, Hkv, Nq, cache, d, dtype, seed=Nq + 7 * Nk + cache)
    kc[:, :, Nk:] = float("nan")
    vc[:, :, Nk:] = float("nan")
    scale = 1.0 / math.sqrt(d)
    o, lse = run(q, kc, vc, Nk, causal, scale)
    O, L = attention_f64(q, kc[:, :, :Nk], vc[:, :, :Nk], causal, scale)
    assert_close(o, lse, O, L, dtype, f"kvcache d{d} {dtype} c{causal} Nq{Nq} Nk{Nk} cache{cache}",
                 strict=False)


@pytest.mark.parametrize("d,dtype", [(64, "fp16"), (128, "bf16")])
def test_chunked_prefill_equals_full_causal_attention(d, dtype):
    """1536 tokens as three 512-token chunks, each against the cache prefix up to its own
    end, reproduce causal attention over the whole sequence row for row."""
    B, Hq, Hkv, N, chunk = 1, 4, 2, 1536, 512
    q, k, v = make_fwd_inputs(B, Hq, Hkv, N, N, d, dtype, seed=d)
    scale = 1.0 / math.sqrt(d)
    kd, vd = k.to(DEV), v.to(DEV)
    outs, lses = [], []
    for i in range(0, N, chunk):
        o, lse = fa.fwd_kvcache(q[:, :, i:i + chunk].contiguous().to(DEV), kd, vd, i + chunk,
                                causal=True, scale=scale)
        outs.append(o)
        lses.append(lse)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    o = torch.cat(outs, dim=2).cpu()
    lse = torch.cat(lses, dim=2).cpu()
    O, L = attention_f64(q, k, v, True, scale)
    assert_close(o, lse, O, L, dtype, f"chunked prefill d{d} {dtype}", strict=False)
