"""Float64 CPU oracle for exact attention.

TEST INFRASTRUCTURE ONLY: imported by `tests/`, `__graft_entry__.smoke()` and the
CPU-baseline leg of `bench.py`, never by the CUDA library or its Python binding.
"""
from .attention import (attention_f64, attention_rows_f64, attention_varlen_f64, decode_f64,
                        visible_mask)
from .backward import attention_bwd_f64
from .paged import (attention_paged_rows_f64, attention_paged_varlen_f64, decode_paged_f64,
                    gather_pages)
from .fp8 import attention_fp8_f64, attention_fp8_rows_f64, e4m3_to_f64
from .tiled import split_kv_decode_f64, tiled_attention_bwd_f64, tiled_attention_f64

__all__ = ["attention_f64", "attention_rows_f64", "decode_f64", "visible_mask",
           "tiled_attention_f64", "tiled_attention_bwd_f64", "split_kv_decode_f64", "attention_bwd_f64", "decode_paged_f64",
           "attention_paged_rows_f64", "gather_pages", "e4m3_to_f64", "attention_fp8_f64",
           "attention_fp8_rows_f64", "attention_varlen_f64", "attention_paged_varlen_f64"]
