"""Plain float64 CPU oracle for attention over a paged KV cache.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this module: only
`tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py` use it.
It shares no code with the CUDA library.

The pages keep a per-session key/value cache that later requests reuse and that is freed
per session (page "Flash Attention ... IO-aware exact" (fr), section on the KV cache and
persistent attention: a cache keyed by session, extended when new tokens arrive and
invalidated per session). On the device that cache is a pool of fixed-size pages shared
by all sessions; a session owns a list of pages (its block-table row), so freeing one
session moves no other session's data. The attention result is unchanged by where the
tokens live: this oracle first gathers each sequence's keys and values from the pool in
token order and then applies the plain attention definition of `attention.py` to them.

Layout read here (the library's layout):
* pool ``[num_pages, Hkv, page_size, d]``: page p, KV head h holds ``page_size``
  consecutive token rows;
* block table ``[B, max_pages]`` int: token t of sequence b lives in page
  ``table[b, t // page_size]`` at row ``t % page_size``;
* only the table entries that cover the sequence's tokens are read.

Parity pins: `tests/test_oracle_paged.py` checks these functions against a brute-force
per-token softmax, page-permutation invariance, poisoned unused pages and the
contiguous-cache oracle.
"""
from __future__ import annotations

import numpy as np

from .attention import _f64, attention_rows_f64, attention_varlen_f64, decode_f64

__all__ = ["gather_pages", "decode_paged_f64", "attention_paged_rows_f64",
           "attention_paged_varlen_f64"]


def gather_pages(pool, table_row, n_tokens: int, page_size: int) -> np.ndarray:
    """Tokens [0, n_tokens) of one sequence, in order: float64 [Hkv, n_tokens, d]."""
    pool = _f64(pool)
    Hkv, d = pool.shape[1], pool.shape[3]
    table_row = np.asarray(table_row, dtype=np.int64)
    out = np.zeros((Hkv, n_tokens, d), dtype=np.float64)
    n_pages = (n_tokens + page_size - 1) // page_size
    for j in range(n_pages):
        t0 = j * page_size
        t1 = min(n_tokens, t0 + page_size)
        out[:, t0:t1] = pool[int(table_row[j]), :, : t1 - t0]
    return out


def decode_paged_f64(q, kpool, vpool, block_table, kv_lens, page_size: int, scale: float):
    """Single-token decode over a paged cache. q: [B,Hq,d]; pools [P,Hkv,page_size,d];
    block_table [B, max_pages]; kv_lens [B]. Returns O [B,Hq,d] and LSE [B,Hq] (float64)."""
    B = q.shape[0]
    lens = np.asarray(_f64(kv_lens), dtype=np.int64)
    table = np.asarray(_f64(block_table), dtype=np.int64)
    O = np.zeros((B, q.shape[1], q.shape[2]), dtype=np.float64)
    L = np.full((B, q.shape[1]), -np.inf, dtype=np.float64)
    for b in range(B):
        n = int(lens[b])
        if n <= 0:
            continue
        K = gather_pages(kpool, table[b], n, page_size)[None]
        V = gather_pages(vpool, table[b], n, page_size)[None]
        o, l = decode_f64(_f64(q[b])[None], K, V, np.array([n]), scale)
        O[b], L[b] = o[0], l[0]
    return O, L


def attention_paged_rows_f64(q, kpool, vpool, block_table, Nk: int, page_size: int,
                             causal: bool, scale: float, b: int, h: int, rows):
    """O and LSE of selected query rows of (batch b, query head h) whose Nk keys and
    values sit in a paged cache (bottom-right causal alignment when Nq != Nk)."""
    table = np.asarray(_f64(block_table), dtype=np.int64)
    K = gather_pages(kpool, table[b], Nk, page_size)[None]
    V = gather_pages(vpool, table[b], Nk, page_size)[None]
    Q = _f64(q[b])[None]
    return attention_rows_f64(Q, K, V, causal, scale, 0, h, rows)


def attention_paged_varlen_f64(q, kpool, vpool, block_table, q_lens, kv_lens, page_size: int,
                               causal: bool, scale: float):
    """Sequences of different lengths over a paged cache: sequence b's first kv_lens[b]
    tokens are gathered through its table row, then `attention_varlen_f64` applies (its
    first q_lens[b] query rows, mask aligned to its own end). Returns O [B,Hq,Nq,d] and LSE
    [B,Hq,Nq], NaN past q_lens[b]."""
    B, Hq, Nq, d = q.shape
    Hkv = kpool.shape[1]
    table = np.asarray(_f64(block_table), dtype=np.int64)
    qn = np.asarray(_f64(q_lens), dtype=np.int64)
    kn = np.asarray(_f64(kv_lens), dtype=np.int64)
    O = np.full((B, Hq, Nq, d), np.nan, dtype=np.float64)
    L = np.full((B, Hq, Nq), np.nan, dtype=np.float64)
    for b in range(B):
        nk = int(kn[b])
        K = gather_pages(kpool, table[b], nk, page_size)[None] if nk > 0 else np.zeros((1, Hkv, 0, d))
        V = gather_pages(vpool, table[b], nk, page_size)[None] if nk > 0 else np.zeros((1, Hkv, 0, d))
        O[b:b + 1], L[b:b + 1] = attention_varlen_f64(_f64(q[b])[None], K, V, qn[b:b + 1],
                                                      kn[b:b + 1], causal, scale)
    return O, L
