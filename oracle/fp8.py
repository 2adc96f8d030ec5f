"""Plain float64 CPU oracle for attention over 8-bit (E4M3) inputs.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this module: only
`tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py` use it.
It shares no code with the CUDA library.

The pages treat lower precision as quantisation of stored values (page "Empreinte
mémoire et calcul des couches Transformer", quantisation bullet: going from 16 to 8 bits
halves the memory). Here Q, K and V are stored as E4M3 codes with one descale factor per
tensor; the real-valued inputs are code value x descale. What the attention computes on
them is the plain definition (see `attention.py`) applied to those real values, so the
oracle decodes every code exactly to float64, multiplies by its descale and calls the
float64 attention definition.

E4M3 as decoded here (the OCP 8-bit floating-point format, E4M3 variant): bit 7 sign,
bits 6..3 exponent with bias 7, bits 2..0 mantissa; exponent 0 encodes subnormals
m/8 x 2^-6; exponent 15 with mantissa 7 is NaN (there are no infinities), so the largest
finite magnitude is 1.75 x 2^8 = 448.

Parity pins: `tests/test_oracle_fp8.py` checks the decoder against closed-form codes and
a library conversion of all 256 codes, and the attention against the float64 oracle on
library-decoded inputs.
"""
from __future__ import annotations

import numpy as np

from .attention import attention_f64, attention_rows_f64

__all__ = ["e4m3_to_f64", "attention_fp8_f64", "attention_fp8_rows_f64"]


def e4m3_to_f64(codes) -> np.ndarray:
    """Exact float64 values of E4M3 codes (uint8 array, or a torch uint8/float8 tensor)."""
    if hasattr(codes, "detach"):
        import torch
        codes = codes.detach().to("cpu")
        if codes.dtype != torch.uint8:
            codes = codes.view(torch.uint8)
        codes = codes.numpy()
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    exp = (c >> 3) & 0xF
    man = c & 0x7
    normal = sign * (1.0 + man / 8.0) * np.exp2(exp - 7.0)
    subnormal = sign * (man / 8.0) * 2.0 ** -6
    out = np.where(exp == 0, subnormal, normal)
    return np.where((exp == 15) & (man == 7), np.nan, out)


def _dequant(codes, descale: float) -> np.ndarray:
    return e4m3_to_f64(codes) * float(descale)


def attention_fp8_f64(q8, k8, v8, q_descale: float, k_descale: float, v_descale: float,
                      causal: bool, scale: float):
    """O [B,Hq,Nq,d] and LSE [B,Hq,Nq] (float64) of the descaled E4M3 inputs."""
    return attention_f64(_dequant(q8, q_descale), _dequant(k8, k_descale),
                         _dequant(v8, v_descale), causal, scale)


def attention_fp8_rows_f64(q8, k8, v8, q_descale: float, k_descale: float, v_descale: float,
                           causal: bool, scale: float, b: int, h: int, rows):
    """Selected query rows of (batch b, query head h); decodes only that head's inputs."""
    Hq, Hkv = q8.shape[1], k8.shape[1]
    kh = h // (Hq // Hkv)
    Q = _dequant(q8[b, h], q_descale)[None, None]
    K = _dequant(k8[b, kh], k_descale)[None, None]
    V = _dequant(v8[b, kh], v_descale)[None, None]
    return attention_rows_f64(Q, K, V, causal, scale, 0, 0, rows)
