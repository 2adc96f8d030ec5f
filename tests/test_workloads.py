"""The five named workloads and the seeded input recipe (CPU only).

The workloads are:
- tiny: non-causal, B=1, H=2, N=128, d=64, fp16;
- mha2k: causal, B=8, H=12 (MHA), N=2048, d=64, fp16;
- gqa8k: causal, B=1, Hq=32, Hkv=8, N=8192, d=128, bf16;
- gqa32k: causal, B=1, Hq=32, Hkv=8, N=32768, d=128, bf16;
- decode: B=64 single-token queries, Hq=32, Hkv=8, d=128, bf16, a contiguous 4096-row
  cache, per-sequence lengths uniform on [512, 4096].

Every workload uses scale 1/sqrt(d) and seed 0. Q, K and V (and the cache) are i.i.d.
N(0, 1) rounded to the 16-bit type; the same seed gives the same tensors.
"""
import math

import numpy as np
import pytest
import torch

from workloads import WORKLOADS, make_decode_inputs, make_fwd_inputs

EXPECTED = {
    "tiny": ("fwd", 1, 2, 2, 128, 64, "fp16", False),
    "mha2k": ("fwd", 8, 12, 12, 2048, 64, "fp16", True),
    "gqa8k": ("fwd", 1, 32, 8, 8192, 128, "bf16", True),
    "gqa32k": ("fwd", 1, 32, 8, 32768, 128, "bf16", True),
    "decode": ("decode", 64, 32, 8, 4096, 128, "bf16", False),
}


def test_the_five_workloads():
    assert set(WORKLOADS) == set(EXPECTED)
    for name, (kind, B, Hq, Hkv, N, d, dtype, causal) in EXPECTED.items():
        w = WORKLOADS[name]
        assert (w.kind, w.B, w.Hq, w.Hkv, w.N, w.d, w.dtype, w.causal) == \
            (kind, B, Hq, Hkv, N, d, dtype, causal), name
        assert w.seed == 0 and w.scale == 1.0 / math.sqrt(d)
    dec = WORKLOADS["decode"]
    assert (dec.kv_len_lo, dec.kv_len_hi) == (512, 4096)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_inputs_are_seeded_standard_normal(dtype):
    q, k, v = make_fwd_inputs(2, 4, 2, 256, 256, 64, dtype, seed=0)
    assert q.dtype == {"fp16": torch.float16, "bf16": torch.bfloat16}[dtype]
    assert q.shape == (2, 4, 256, 64) and k.shape == v.shape == (2, 2, 256, 64)
    for t in (q, k, v):
        x = t.float().numpy().ravel()
        assert abs(x.mean()) < 0.02 and abs(x.std() - 1.0) < 0.02     # 65536 draws or more
    q2, k2, v2 = make_fwd_inputs(2, 4, 2, 256, 256, 64, dtype, seed=0)
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)
    q3, _, _ = make_fwd_inputs(2, 4, 2, 256, 256, 64, dtype, seed=1)
    assert not torch.equal(q, q3)


def test_decode_lengths_cover_their_range():
    w = WORKLOADS["decode"]
    lens, q, kc, vc = make_decode_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.dtype, w.kv_len_lo,
                                         w.kv_len_hi, w.seed)
    assert lens.dtype == torch.int32 and lens.shape == (64,)
    assert q.shape == (64, 32, 128) and kc.shape == vc.shape == (64, 8, 4096, 128)
    n = lens.numpy()
    assert n.min() >= 512 and n.max() <= 4096
    # Uniform on [512, 4096]: mean 2304, standard deviation about 1035; 64 draws put the
    # sample mean within 4 standard errors (about 520) of it.
    assert abs(n.mean() - 2304) < 520
    big = make_decode_inputs(4096, 1, 1, 8, 8, "bf16", 512, 4096, seed=3)[0].numpy()
    assert big.min() == 512 and big.max() == 4096        # both ends are drawn
    assert abs(np.median(big) - 2304) < 120
