"""Plain float64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this module: only
`tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py` use it.
It shares no code with the CUDA library.

What it computes is the plain definition of attention, written out untiled:
``O = softmax(scale * Q K^T) V`` with ``scale = 1/sqrt(d)`` in every workload (page
"Kotaemon FlashAttention", the attention formula; page "Flash Attention ... IO-aware
exact" (fr), tiling pseudo-code, where the scores are divided by sqrt(d)). The tiled
method on those pages reaches exactly this result up to rounding (page "Kotaemon
FlashAttention", algorithm bullets and the exactness paragraph), so the oracle is the
definition itself, not the tiled algorithm.

Readings taken where the pages are silent or garbled:

* the second output ``L`` returned by the pages' pseudo-code is the per-row logsumexp,
  natural log, of the *scaled* scores: ``LSE_i = log(sum_j exp(scale * q_i . k_j))``;
* causal masking with Nq != Nk is bottom-right aligned: key j is visible to query i iff
  ``j <= i + (Nk - Nq)`` (page "Flash Attention ... IO-aware exact" (fr), manual chunking
  example: a query chunk ending at token t attends to all keys up to t);
* a row with no visible key has ``O = 0`` and ``LSE = -inf``;
* grouped-query attention maps query head h to KV head ``h // (Hq // Hkv)``;
* inputs are 16-bit values upcast exactly to float64.

The softmax is taken in two passes over the materialised score row: the row maximum
first, then the exponentials and their sum.

Parity pins: every function here is pinned by `tests/test_oracle_pins.py` against
closed forms, brute force, a library special case and hand-worked fixtures.
"""
from __future__ import annotations

import numpy as np

__all__ = ["attention_f64", "attention_rows_f64", "attention_varlen_f64", "decode_f64",
           "visible_mask"]


def _f64(x) -> np.ndarray:
    """Exact upcast of a numpy array or CPU torch tensor (fp16/bf16/fp32/fp64) to float64."""
    if hasattr(x, "detach"):  # torch tensor: bf16 has no numpy dtype, go through float32
        import torch
        x = x.detach().to("cpu")
        if x.dtype in (torch.float16, torch.bfloat16):
            x = x.to(torch.float32)
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def visible_mask(rows: np.ndarray, Nq: int, Nk: int, causal: bool) -> np.ndarray:
    """Boolean [len(rows), Nk]: True where key j is visible to query row i."""
    cols = np.arange(Nk)[None, :]
    if not causal:
        return np.ones((len(rows), Nk), dtype=bool)
    return cols <= (np.asarray(rows)[:, None] + (Nk - Nq))


def _softmax_rows(S: np.ndarray, vis: np.ndarray, V: np.ndarray):
    """Two-pass softmax of the score rows S (masked by vis), then P.V and the row LSE."""
    S = np.where(vis, S, -np.inf)
    m = S.max(axis=1)                                   # pass 1: row maximum
    has = np.isfinite(m)
    m_safe = np.where(has, m, 0.0)
    E = np.exp(S - m_safe[:, None])                     # pass 2: exponentials (0 where masked)
    l = E.sum(axis=1)
    O = np.zeros((S.shape[0], V.shape[1]), dtype=np.float64)
    O[has] = (E[has] / l[has, None]) @ V
    lse = np.full(S.shape[0], -np.inf, dtype=np.float64)
    lse[has] = m[has] + np.log(l[has])
    return O, lse


def attention_rows_f64(q, k, v, causal: bool, scale: float, b: int, h: int, rows):
    """O and LSE for selected query rows of one (batch b, query head h).

    q: [B,Hq,Nq,d]; k, v: [B,Hkv,Nk,d]. Returns (O [len(rows), d], LSE [len(rows)]).
    """
    Hq, Nq = q.shape[1], q.shape[2]
    Hkv, Nk = k.shape[1], k.shape[2]
    g = Hq // Hkv
    rows = np.asarray(rows, dtype=np.int64)
    Q = _f64(q[b, h])[rows]
    K = _f64(k[b, h // g])
    V = _f64(v[b, h // g])
    S = scale * (Q @ K.T)
    return _softmax_rows(S, visible_mask(rows, Nq, Nk, causal), V)


def attention_f64(q, k, v, causal: bool, scale: float):
    """Full oracle: O [B,Hq,Nq,d] float64 and LSE [B,Hq,Nq] float64."""
    B, Hq, Nq, d = q.shape
    O = np.zeros((B, Hq, Nq, d), dtype=np.float64)
    L = np.zeros((B, Hq, Nq), dtype=np.float64)
    rows = np.arange(Nq)
    for b in range(B):
        for h in range(Hq):
            O[b, h], L[b, h] = attention_rows_f64(q, k, v, causal, scale, b, h, rows)
    return O, L


def decode_f64(q, kcache, vcache, kv_lens, scale: float):
    """Single-token decode over a KV cache: the same definition with Nq = 1, non-causal,
    over cache rows [0, kv_lens[b]).

    q: [B,Hq,d]; kcache, vcache: [B,Hkv,cache_len,d]; kv_lens: [B] ints.
    Returns O [B,Hq,d] and LSE [B,Hq] (float64).
    """
    B, Hq, d = q.shape
    Hkv = kcache.shape[1]
    g = Hq // Hkv
    lens = np.asarray(_f64(kv_lens), dtype=np.int64)
    O = np.zeros((B, Hq, d), dtype=np.float64)
    L = np.full((B, Hq), -np.inf, dtype=np.float64)
    for b in range(B):
        n = int(lens[b])
        if n <= 0:
            continue
        for h in range(Hq):
            Qh = _f64(q[b, h])[None, :]
            K = _f64(kcache[b, h // g, :n])
            V = _f64(vcache[b, h // g, :n])
            S = scale * (Qh @ K.T)
            o, l = _softmax_rows(S, np.ones_like(S, dtype=bool), V)
            O[b, h], L[b, h] = o[0], l[0]
    return O, L


def attention_varlen_f64(q, k, v, q_lens, kv_lens, causal: bool, scale: float):
    """Sequences of different lengths in one batch: sequence b has q_lens[b] query rows (the
    first rows of q[b]) and kv_lens[b] keys and values (the first rows of k[b], v[b]), and
    is its own attention problem, its causal mask aligned to its own end (key j visible to
    query i iff j <= i + kv_lens[b] - q_lens[b]). This is the per-session cache of page
    "Flash Attention ... IO-aware exact" (fr), KV-cache section (each session holds its own
    number of tokens), with the plain definition applied to each session.

    q: [B,Hq,Nq,d]; k, v: [B,Hkv,Nk,d]; lengths within [0, Nq] and [0, Nk]. Returns O
    [B,Hq,Nq,d] and LSE [B,Hq,Nq] (float64); rows past q_lens[b] are NaN (no result)."""
    B, Hq, Nq, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    qn = np.asarray(_f64(q_lens), dtype=np.int64)
    kn = np.asarray(_f64(kv_lens), dtype=np.int64)
    O = np.full((B, Hq, Nq, d), np.nan, dtype=np.float64)
    L = np.full((B, Hq, Nq), np.nan, dtype=np.float64)
    for b in range(B):
        nq, nk = int(qn[b]), int(kn[b])
        if nq <= 0:
            continue
        rows = np.arange(nq)
        for h in range(Hq):
            if nk <= 0:
                O[b, h, :nq] = 0.0
                L[b, h, :nq] = -np.inf
                continue
            Q = _f64(q[b, h])[:nq]
            K = _f64(k[b, h // g])[:nk]
            V = _f64(v[b, h // g])[:nk]
            S = scale * (Q @ K.T)
            O[b, h, :nq], L[b, h, :nq] = _softmax_rows(S, visible_mask(rows, nq, nk, causal), V)
    return O, L
