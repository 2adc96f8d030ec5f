"""Seeded synthetic inputs for exact-attention workloads.

This module holds no attention arithmetic: it only draws random tensors and describes
the five workload shapes. It is shared by the tests, the benchmark and the smoke check;
neither the CUDA library nor the CPU oracle imports it.

Recipe (one `torch.Generator` seeded with the workload's seed, CPU side):

* decode workloads draw the per-sequence KV lengths first, as
  ``torch.randint(lo, hi + 1, (B,))`` (int32), uniform on ``[lo, hi]`` inclusive;
* then Q, K, V in that order, each as ``torch.randn(shape, float32)`` rounded
  (round-to-nearest-even) to fp16 or bf16. Large tensors are drawn in chunks along
  their leading (batch) axis, always in the same order, so the stream of draws is fixed.

Shapes follow the pages' workloads: page "Flash Attention ... IO-aware exact" (fr),
PyTorch section (batch 8, 12 heads, 2048 tokens, head dim 64, fp16, causal); page
"Empreinte mémoire et calcul des couches Transformer", KV-cache paragraph (8 KV heads
for grouped-query attention, head dim 128, 32 layers, 4096-token caches); page
"Kotaemon FlashAttention", HuggingFace example (8B-class Llama in bf16).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

__all__ = ["Workload", "WORKLOADS", "make_fwd_inputs", "make_decode_inputs",
           "make_page_table", "paginate", "make_fp8_inputs", "fwd_flops", "decode_kv_bytes",
           "torch_dtype"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "fwd" or "decode"
    B: int
    Hq: int
    Hkv: int
    N: int               # sequence length (fwd) or cache capacity (decode)
    d: int
    dtype: str           # "fp16" or "bf16"
    causal: bool
    kv_len_lo: int = 0   # decode only
    kv_len_hi: int = 0   # decode only
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def describe(self) -> str:
        if self.kind == "decode":
            return (f"GQA decode B={self.B} Hq={self.Hq} Hkv={self.Hkv} d={self.d} {self.dtype} "
                    f"cache={self.N} kv_len~U[{self.kv_len_lo},{self.kv_len_hi}] seed={self.seed}")
        heads = f"H={self.Hq}" if self.Hq == self.Hkv else f"Hq={self.Hq} Hkv={self.Hkv}"
        return (f"{'causal' if self.causal else 'non-causal'} attention B={self.B} {heads} "
                f"N={self.N} d={self.d} {self.dtype} seed={self.seed}")


WORKLOADS = {
    "tiny": Workload("tiny", "fwd", 1, 2, 2, 128, 64, "fp16", False),
    "mha2k": Workload("mha2k", "fwd", 8, 12, 12, 2048, 64, "fp16", True),
    "gqa8k": Workload("gqa8k", "fwd", 1, 32, 8, 8192, 128, "bf16", True),
    "gqa32k": Workload("gqa32k", "fwd", 1, 32, 8, 32768, 128, "bf16", True),
    "decode": Workload("decode", "decode", 64, 32, 8, 4096, 128, "bf16", False, 512, 4096),
}


def torch_dtype(name: str) -> torch.dtype:
    return {"fp16": torch.float16, "bf16": torch.bfloat16}[name]


def _randn16(gen: torch.Generator, shape, dtype: torch.dtype) -> torch.Tensor:
    """Draw N(0,1) float32 in chunks along axis 0 and round each chunk to `dtype`."""
    out = torch.empty(shape, dtype=dtype)
    for i in range(shape[0]):
        out[i] = torch.randn(shape[1:], generator=gen, dtype=torch.float32).to(dtype)
    return out


def make_fwd_inputs(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int, dtype: str,
                    seed: int = 0):
    """Q [B,Hq,Nq,d], K and V [B,Hkv,Nk,d]; CPU tensors of the 16-bit dtype."""
    gen = torch.Generator().manual_seed(seed)
    dt = torch_dtype(dtype)
    q = _randn16(gen, (B, Hq, Nq, d), dt)
    k = _randn16(gen, (B, Hkv, Nk, d), dt)
    v = _randn16(gen, (B, Hkv, Nk, d), dt)
    return q, k, v


def make_decode_inputs(B: int, Hq: int, Hkv: int, cache_len: int, d: int, dtype: str,
                       kv_len_lo: int, kv_len_hi: int, seed: int = 0,
                       kv_lens: Optional[torch.Tensor] = None):
    """kv_lens int32 [B], q [B,Hq,d], kcache and vcache [B,Hkv,cache_len,d] (CPU)."""
    gen = torch.Generator().manual_seed(seed)
    dt = torch_dtype(dtype)
    drawn = torch.randint(kv_len_lo, kv_len_hi + 1, (B,), generator=gen, dtype=torch.int64)
    if kv_lens is None:
        kv_lens = drawn
    kv_lens = kv_lens.to(torch.int32)
    q = _randn16(gen, (B, Hq, d), dt)
    kc = _randn16(gen, (B, Hkv, cache_len, d), dt)
    vc = _randn16(gen, (B, Hkv, cache_len, d), dt)
    return kv_lens, q, kc, vc


def make_fp8_inputs(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int, seed: int = 0):
    """E4M3 Q [B,Hq,Nq,d], K and V [B,Hkv,Nk,d] as uint8 codes, and their descales.

    Q, K, V are drawn as in `make_fwd_inputs` (N(0,1) float32, in that order, chunked along
    the batch axis), then each tensor is divided by descale = amax / 448 (its largest
    magnitude lands on the largest finite E4M3 value) and rounded to E4M3 (round to
    nearest even) by torch's float8_e4m3fn conversion. Returns
    (q8, k8, v8, q_descale, k_descale, v_descale), CPU tensors and Python floats.
    """
    gen = torch.Generator().manual_seed(seed)
    out = []
    for shape in ((B, Hq, Nq, d), (B, Hkv, Nk, d), (B, Hkv, Nk, d)):
        x = torch.empty(shape, dtype=torch.float32)
        for i in range(shape[0]):
            x[i] = torch.randn(shape[1:], generator=gen, dtype=torch.float32)
        descale = float(x.abs().max()) / 448.0
        out.append(((x / descale).to(torch.float8_e4m3fn).view(torch.uint8), descale))
    (q8, dq), (k8, dk), (v8, dv) = out
    return q8, k8, v8, dq, dk, dv


def make_page_table(lens, page_size: int, max_pages: int, spare_pages: int = 3, seed: int = 0,
                    fill: int = -1):
    """Random page assignment for a paged KV cache.

    Sequence b receives ceil(lens[b] / page_size) pages, taken in order from one seeded
    random permutation of the pool (``torch.randperm``), so pages of different sequences
    never coincide and consecutive tokens land in scattered pages. The pool has
    ``spare_pages`` pages more than the sequences use; table entries past a sequence's
    last page hold ``fill``. Returns (table int32 [B, max_pages], num_pages).
    """
    lens = [int(x) for x in torch.as_tensor(lens).tolist()]
    need = [(n + page_size - 1) // page_size for n in lens]
    if max(need, default=0) > max_pages:
        raise ValueError("a sequence needs more pages than max_pages")
    num_pages = sum(need) + spare_pages
    gen = torch.Generator().manual_seed(seed)
    perm = torch.randperm(num_pages, generator=gen).to(torch.int32)
    table = torch.full((len(lens), max_pages), fill, dtype=torch.int32)
    at = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[at:at + n]
        at += n
    return table, num_pages


def paginate(cache: torch.Tensor, table: torch.Tensor, lens, page_size: int, num_pages: int,
             fill_value: float = float("nan")) -> torch.Tensor:
    """Copy tokens [0, lens[b]) of a contiguous cache [B, Hkv, L, d] into a page pool
    [num_pages, Hkv, page_size, d] laid out by `table` (token t of sequence b goes to
    page table[b, t // page_size], row t % page_size). Pool rows no token maps to hold
    `fill_value` (NaN by default, so a kernel that reads them shows it)."""
    B, Hkv, _, d = cache.shape
    pool = torch.full((num_pages, Hkv, page_size, d), fill_value, dtype=cache.dtype)
    lens = [int(x) for x in torch.as_tensor(lens).tolist()]
    for b in range(B):
        for j in range((lens[b] + page_size - 1) // page_size):
            t0 = j * page_size
            t1 = min(lens[b], t0 + page_size)
            pool[int(table[b, j]), :, : t1 - t0] = cache[b, :, t0:t1]
    return pool


def workload_inputs(w: Workload):
    if w.kind == "decode":
        return make_decode_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.dtype, w.kv_len_lo,
                                  w.kv_len_hi, w.seed)
    return make_fwd_inputs(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, w.seed)


def fwd_flops(B: int, Hq: int, Nq: int, Nk: int, d: int, causal: bool) -> float:
    """Algorithmic FLOPs: 4*d per visible (query, key) pair (QK^T and PV, 2 flops per MAC).

    Causal counts visible pairs under the bottom-right alignment (key j visible to query
    i iff j <= i + Nk - Nq); for Nq == Nk that is N(N+1)/2 pairs per head.
    """
    if causal:
        off = Nk - Nq
        pairs = 0
        for i in range(Nq):
            pairs += max(0, min(Nk, i + off + 1))
    else:
        pairs = Nq * Nk
    return 4.0 * d * pairs * B * Hq


def decode_kv_bytes(kv_lens, Hkv: int, d: int, elem_bytes: int = 2) -> int:
    """Bytes of K and V a decode step must read: 2 * Hkv * d * elem * sum(kv_len)."""
    total = int(torch.as_tensor(kv_lens).to(torch.int64).sum())
    return 2 * Hkv * d * elem_bytes * total
