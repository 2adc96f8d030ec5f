"""Plain float64 CPU oracle for the gradients of exact attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this module: only
`tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py` use it.
It shares no code with the CUDA library.

The pages describe the backward pass only as recomputation: the tiled method keeps no
N x N matrix, so the backward pass recomputes the scores tile by tile from Q, K and the
saved per-row statistic L instead of storing them (page "Flash Attention" (zh), "IO 感知
的算法设计", tiling plus recomputation; page "Flash Attention ... IO-aware exact" (fr),
the pseudo-code's second output L). What the backward pass computes is therefore fixed by
the forward definition alone: the gradients of O = softmax(scale * Q K^T) V with respect
to Q, K and V for an upstream gradient dO. This module writes that derivative out
untiled, per (batch, query head):

    S = scale * Q K^T   (masked entries: -inf)      P = softmax(S) row by row
    dV = P^T dO         dP = dO V^T                  D_i = sum_j P_ij dP_ij
    dS = P * (dP - D)   dQ = scale * dS K            dK = scale * dS^T Q

Readings taken:
* masking and grouped-query mapping are the forward oracle's (bottom-right causal; query
  head h reads KV head h // (Hq // Hkv)); a KV head's dK and dV sum the contributions of
  all query heads that read it;
* a row with no visible key has P = 0, so it contributes nothing to any gradient and its
  dQ is 0;
* D_i equals sum_d dO_id O_id (the identity the recomputed backward pass uses); the oracle
  takes it from P and dP directly.

Parity pins: `tests/test_oracle_bwd.py` checks these functions against central finite
differences of the forward oracle, closed-form invariants and the grouped-query sum.
"""
from __future__ import annotations

import numpy as np

from .attention import _f64, visible_mask

__all__ = ["attention_bwd_f64"]


def _head_bwd(Q, K, V, dO, vis, scale):
    """Gradients of one (batch, query head) problem. All arrays float64."""
    S = np.where(vis, scale * (Q @ K.T), -np.inf)
    m = S.max(axis=1)
    has = np.isfinite(m)
    E = np.zeros_like(S)
    E[has] = np.exp(S[has] - m[has, None])
    l = E.sum(axis=1)
    P = np.zeros_like(S)
    P[has] = E[has] / l[has, None]
    dV = P.T @ dO
    dP = dO @ V.T
    D = (P * dP).sum(axis=1)
    dS = P * (dP - D[:, None])
    dQ = scale * (dS @ K)
    dK = scale * (dS.T @ Q)
    return dQ, dK, dV


def attention_bwd_f64(q, k, v, do, causal: bool, scale: float):
    """dQ [B,Hq,Nq,d], dK and dV [B,Hkv,Nk,d], float64, for upstream gradient do [B,Hq,Nq,d]."""
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    g = Hq // Hkv
    dq = np.zeros((B, Hq, Nq, d), dtype=np.float64)
    dk = np.zeros((B, Hkv, Nk, d), dtype=np.float64)
    dv = np.zeros((B, Hkv, Nk, d), dtype=np.float64)
    vis = visible_mask(np.arange(Nq), Nq, Nk, causal)
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            dQ, dK, dV = _head_bwd(_f64(q[b, h]), _f64(k[b, kh]), _f64(v[b, kh]), _f64(do[b, h]),
                                   vis, scale)
            dq[b, h] = dQ
            dk[b, kh] += dK
            dv[b, kh] += dV
    return dq, dk, dv
