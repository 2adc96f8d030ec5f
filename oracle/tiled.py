"""Tiled online-softmax attention, its backward pass by tile-wise recomputation, and
split-KV decode merged by the chunks' LSEs, in plain float64 Python, for tiny inputs.

TEST INFRASTRUCTURE ONLY (see `oracle/attention.py`). It exists to check the pages'
exactness claim: processing the keys tile by tile with a running maximum and a running
normaliser gives the same result as the untiled definition (page "Kotaemon
FlashAttention", algorithm bullets: Q split into row blocks, K_j/V_j blocks loaded per
row block, running max and normaliser updated, result identical to the original).

The loop is derived from the online-softmax recurrence (page "Flash Attention" (zh),
online-softmax bullet; page "Kotaemon FlashAttention", running max and normaliser): query
rows in blocks of Br, keys in blocks of Bc inside each row block, and for every key tile

    m_new = max(m, rowmax(S_ij));  alpha = exp(m - m_new)
    P_ij  = exp(S_ij - m_new);     l = alpha * l + rowsum(P_ij)
    O_i   = alpha * O_i + P_ij V_j

and after the last tile ``O_i / l`` and ``L_i = m + log(l)``. Tr = ceil(Nq/Br),
Tc = ceil(Nk/Bc); masked scores are -inf.

Two optional arguments restate the kernels' departures from that recurrence, both of which
cancel in O / l (the properties check that they do, for any tile sizes):

* ``tau`` (log2 units, >= 0): a lazy running maximum. A row's m moves to the tile's
  maximum only when that maximum exceeds m by more than tau * ln 2; otherwise m, l and O
  keep their scale and P_ij = exp(S_ij - m) may reach 2^tau. tau = 0 is the recurrence
  above. The 16-bit kernels use 8, the E4M3 kernel 4.
* ``offset`` (log2 units): P_ij = exp(S_ij - m + offset * ln 2), and the offset is taken
  back out of L. The E4M3 kernel uses 4, so that P stays in E4M3's normal range.

Prior art, not followed: the tiling pseudo-code of page "Flash Attention ... IO-aware
exact" (fr) has the same outer loop over Q_i and returns O and L, but it has no loop over
j, leaves Tr undefined and applies a separate softmax to each tile before a plain ``+=``,
which is not exact; this code does not take that form.
"""
from __future__ import annotations

import numpy as np

from .attention import _f64, visible_mask

__all__ = ["tiled_attention_f64", "tiled_attention_bwd_f64", "split_kv_decode_f64"]


def tiled_attention_f64(Q, K, V, causal: bool, scale: float, Br: int, Bc: int,
                        tau: float = 0.0, offset: float = 0.0):
    """One head: Q [Nq,d], K and V [Nk,d]. Returns O [Nq,d] and L [Nq] (float64)."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    Nq, d = Q.shape
    Nk = K.shape[0]
    Tr = -(-Nq // Br)
    Tc = -(-Nk // Bc)
    O = np.zeros((Nq, d))
    L = np.full(Nq, -np.inf)
    tau_ln, off_ln = tau * np.log(2.0), offset * np.log(2.0)
    for i in range(Tr):
        r0, r1 = i * Br, min(Nq, (i + 1) * Br)
        Qi = Q[r0:r1]
        Oi = np.zeros((r1 - r0, d))
        li = np.zeros(r1 - r0)
        mi = np.full(r1 - r0, -np.inf)
        for j in range(Tc):
            c0, c1 = j * Bc, min(Nk, (j + 1) * Bc)
            Kj, Vj = K[c0:c1], V[c0:c1]
            Sij = scale * (Qi @ Kj.T)
            vis = visible_mask(np.arange(r0, r1), Nq, Nk, causal)[:, c0:c1]
            Sij = np.where(vis, Sij, -np.inf)
            tmax = Sij.max(axis=1)
            m_new = np.where(tmax > mi + tau_ln, tmax, mi)    # tau = 0: max(m, rowmax)
            ref = np.where(np.isfinite(m_new), m_new, 0.0)   # rows with nothing visible yet
            alpha = np.where(np.isfinite(mi), np.exp(mi - ref), 0.0)
            Pij = np.exp(Sij - ref[:, None] + off_ln)
            li = alpha * li + Pij.sum(axis=1)
            Oi = alpha[:, None] * Oi + Pij @ Vj
            mi = m_new
        seen = li > 0
        O[r0:r1][seen] = Oi[seen] / li[seen, None]
        L[r0:r1][seen] = mi[seen] + np.log(li[seen]) - off_ln
    return O, L


def tiled_attention_bwd_f64(Q, K, V, dO, O, L, causal: bool, scale: float, Br: int, Bc: int):
    """One head's gradients by tile-wise recomputation, float64: (dQ [Nq,d], dK, dV [Nk,d]).

    This restates the backward pass the way the tiled method runs it (page "Flash
    Attention" (zh), "IO 感知的算法设计": no N x N matrix is kept, so the scores are
    recomputed tile by tile from Q, K and the saved per-row statistic L). O and L are the
    forward's outputs. First D_i = sum_c dO_ic O_ic for every row (equal to
    sum_j P_ij dP_ij because O = P V); then, for every key tile j of Bc keys and every
    query tile i of Br rows:

        S_ij  = scale * Q_i K_j^T (masked: -inf)     P_ij = exp(S_ij - L_i)
        dV_j += P_ij^T dO_i                          dP_ij = dO_i V_j^T
        dS_ij = P_ij * (dP_ij - D_i)
        dQ_i += scale * dS_ij K_j                    dK_j += scale * dS_ij^T Q_i

    A row with L_i = -inf (no visible key) has P = 0 and contributes nothing."""
    Q, K, V, dO, O, L = _f64(Q), _f64(K), _f64(V), _f64(dO), _f64(O), _f64(L)
    Nq, d = Q.shape
    Nk = K.shape[0]
    D = (dO * O).sum(axis=1)
    Lf = np.where(np.isfinite(L), L, np.inf)          # exp(-inf - inf) = 0 for empty rows
    dQ = np.zeros((Nq, d))
    dK = np.zeros((Nk, d))
    dV = np.zeros((Nk, d))
    for j in range(-(-Nk // Bc)):
        c0, c1 = j * Bc, min(Nk, (j + 1) * Bc)
        Kj, Vj = K[c0:c1], V[c0:c1]
        for i in range(-(-Nq // Br)):
            r0, r1 = i * Br, min(Nq, (i + 1) * Br)
            vis = visible_mask(np.arange(r0, r1), Nq, Nk, causal)[:, c0:c1]
            Sij = np.where(vis, scale * (Q[r0:r1] @ Kj.T), -np.inf)
            Pij = np.exp(Sij - Lf[r0:r1, None])
            dV[c0:c1] += Pij.T @ dO[r0:r1]
            dPij = dO[r0:r1] @ Vj.T
            dSij = Pij * (dPij - D[r0:r1, None])
            dQ[r0:r1] += scale * (dSij @ Kj)
            dK[c0:c1] += scale * (dSij.T @ Q[r0:r1])
    return dQ, dK, dV


def split_kv_decode_f64(q, K, V, bounds, scale: float):
    """One decode head over keys split into chunks, then merged by their LSEs (float64).

    q [d]; K and V [n, d]; bounds: 0 = b_0 <= b_1 <= ... <= b_S = n, chunk s holding keys
    [b_s, b_{s+1}) (a chunk may be empty). Each chunk is its own attention problem, giving
    a partial O_s and LSE_s (an empty chunk gives O_s = 0, LSE_s = -inf); the merge is

        LSE = log sum_s exp(LSE_s)        O = sum_s exp(LSE_s - LSE) O_s

    which is exact because the softmax normaliser is a sum over keys, the same
    associativity the online-softmax update uses (page "Kotaemon FlashAttention",
    exactness paragraph: the block-wise result is identical to the original). Returns
    (O [d], LSE); no keys at all gives O = 0, LSE = -inf."""
    q, K, V = _f64(q), _f64(K), _f64(V)
    bounds = [int(x) for x in bounds]
    parts = []
    for s0, s1 in zip(bounds[:-1], bounds[1:]):
        if s1 <= s0:
            parts.append((np.zeros(V.shape[1]), -np.inf))
            continue
        sc = scale * (K[s0:s1] @ q)
        m = sc.max()
        e = np.exp(sc - m)
        parts.append(((e @ V[s0:s1]) / e.sum(), m + np.log(e.sum())))
    lses = np.array([l for _, l in parts])
    if not np.isfinite(lses).any():
        return np.zeros(V.shape[1]), -np.inf
    mx = lses[np.isfinite(lses)].max()
    lse = mx + np.log(np.sum(np.exp(lses[np.isfinite(lses)] - mx)))
    O = np.zeros(V.shape[1])
    for o_s, l_s in parts:
        if np.isfinite(l_s):
            O += np.exp(l_s - lse) * o_s
    return O, lse
