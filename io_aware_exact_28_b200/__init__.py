"""Python binding of libfa_b200.so: exact attention on B200 (sm_100a).

Argument marshalling only. Every step of the computation runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback. If the shared library is missing or fails
to load, the first call raises `FALibraryError`.

Functions mirror the C ABI in ``include/fa.h``:

* ``fwd(q, k, v, causal, scale)`` -> ``(o, lse)``   (``fa_fwd``)
* ``decode(q, kcache, vcache, kv_lens, scale)`` -> ``(o, lse)``   (``fa_decode``)
* ``decode_workspace_bytes(B, Hq, max_kv_len, d)``   (``fa_decode_workspace_bytes``)
* ``fwd_kvcache``, ``fwd_paged``, ``decode_paged``, ``decode_noalloc``, ``bwd``, ``fwd_fp8``
* ``device_status``, ``set_wait_timeout_ns``, ``debug_skip_q_load``, ``build_info``
"""
from __future__ import annotations

import ctypes
import math
import os
import threading
from typing import Optional, Tuple

__all__ = ["FAError", "FALibraryError", "LIB_PATH", "lib", "fwd", "decode",
           "decode_workspace_bytes", "device_status", "set_wait_timeout_ns",
           "debug_skip_q_load", "build_info", "status_string", "EXPORTED_SYMBOLS",
           "FA_OK", "FA_ERR_INVALID_ARG", "FA_ERR_UNSUPPORTED", "FA_ERR_ALIGNMENT",
           "FA_ERR_CUDA", "FA_ERR_DEVICE_TIMEOUT", "FA_ERR_WORKSPACE", "FA_FP16", "FA_BF16",
           "decode_noalloc", "DECODE_NOALLOC_SCRATCH_BYTES", "fwd_kvcache", "bwd",
           "bwd_workspace_bytes", "fwd_paged", "decode_paged", "fwd_fp8"]

# FA_B200_LIB may name another build of the same library (e.g. a variant for timing).
LIB_PATH = os.environ.get("FA_B200_LIB") or \
    os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa_b200.so")

FA_FP16, FA_BF16 = 0, 1
(FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_CUDA,
 FA_ERR_DEVICE_TIMEOUT, FA_ERR_WORKSPACE) = range(7)

EXPORTED_SYMBOLS = ("fa_fwd", "fa_decode", "fa_decode_workspace_bytes", "fa_status_string",
                    "fa_device_status", "fa_set_wait_timeout_ns", "fa_debug_skip_q_load",
                    "fa_build_info", "fa_decode_noalloc", "fa_fwd_kvcache", "fa_bwd",
                    "fa_bwd_workspace_bytes", "fa_fwd_paged", "fa_decode_paged", "fa_fwd_fp8")

# Size of the library's fixed decode scratch (FA_DECODE_NOALLOC_SCRATCH_BYTES in fa.h).
DECODE_NOALLOC_SCRATCH_BYTES = 32 << 20


class FALibraryError(RuntimeError):
    """The CUDA library could not be loaded (not built, or built for another target)."""


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where} failed: {status_string(status)} ({status})")


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Load libfa_b200.so once and declare the C signatures."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise FALibraryError(
                f"{LIB_PATH} is missing; build it with `python io_aware_exact_28_b200/csrc/build.py`")
        try:
            L = ctypes.CDLL(LIB_PATH)
        except OSError as e:
            raise FALibraryError(f"cannot load {LIB_PATH}: {e}") from e
        c_int, c_float, c_void_p, c_size_t = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
        L.fa_fwd.argtypes = [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p] + [c_int] * 7 + \
            [c_float, c_int, c_void_p]
        L.fa_fwd.restype = c_int
        L.fa_fwd_kvcache.argtypes = [c_void_p] * 7 + [c_int] * 8 + [c_float, c_int, c_void_p]
        L.fa_fwd_kvcache.restype = c_int
        L.fa_bwd.argtypes = [c_void_p] * 9 + [c_int] * 7 + [c_float, c_int, c_void_p, c_size_t, c_void_p]
        L.fa_bwd.restype = c_int
        L.fa_bwd_workspace_bytes.argtypes = [c_int] * 3
        L.fa_bwd_workspace_bytes.restype = c_size_t
        L.fa_decode.argtypes = [c_void_p] * 6 + [c_int] * 5 + [c_float, c_int, c_void_p, c_size_t,
                                                                 c_void_p]
        L.fa_decode.restype = c_int
        L.fa_decode_workspace_bytes.argtypes = [c_int] * 4
        L.fa_decode_workspace_bytes.restype = c_size_t
        L.fa_status_string.argtypes = [c_int]
        L.fa_status_string.restype = ctypes.c_char_p
        L.fa_device_status.argtypes = [c_int]
        L.fa_device_status.restype = c_int
        L.fa_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
        L.fa_set_wait_timeout_ns.restype = None
        L.fa_debug_skip_q_load.argtypes = [c_int]
        L.fa_debug_skip_q_load.restype = None
        L.fa_build_info.argtypes = []
        L.fa_build_info.restype = ctypes.c_char_p
        L.fa_decode_noalloc.argtypes = [c_void_p] * 6 + [c_int] * 5 + [c_float, c_int, c_void_p]
        L.fa_decode_noalloc.restype = c_int
        L.fa_fwd_paged.argtypes = [c_void_p] * 8 + [c_int] * 10 + [c_float, c_int, c_void_p]
        L.fa_fwd_paged.restype = c_int
        L.fa_decode_paged.argtypes = [c_void_p] * 7 + [c_int] * 7 + [c_float, c_int, c_void_p,
                                                                     c_size_t, c_void_p]
        L.fa_decode_paged.restype = c_int
        L.fa_fwd_fp8.argtypes = [c_void_p] * 5 + [c_int] * 7 + [c_float] * 4 + [c_void_p]
        L.fa_fwd_fp8.restype = c_int
        _lib = L
        return L


def status_string(status: int) -> str:
    return lib().fa_status_string(int(status)).decode()


def build_info() -> str:
    return lib().fa_build_info().decode()


def device_status(clear: bool = True) -> int:
    return int(lib().fa_device_status(1 if clear else 0))


def set_wait_timeout_ns(ns: int) -> None:
    lib().fa_set_wait_timeout_ns(int(ns))


def debug_skip_q_load(enable: bool) -> None:
    lib().fa_debug_skip_q_load(1 if enable else 0)


def decode_workspace_bytes(B: int, Hq: int, max_kv_len: int, d: int) -> int:
    return int(lib().fa_decode_workspace_bytes(B, Hq, max_kv_len, d))


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float16:
        return FA_FP16
    if t.dtype == torch.bfloat16:
        return FA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float16 or bfloat16")


def _check(t, name: str, ndim: int, device) -> None:
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_buf(t, name: str, shape, dtype, device) -> None:
    """A caller-supplied tensor whose size the kernels trust (an output, the LSE input of
    the backward pass): exact shape and dtype, on `device`, contiguous."""
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    _check(t, name, len(shape), device)


def _check_workspace(ws, device) -> None:
    """Scratch passed by the caller: device memory on `device`, contiguous (its byte size
    is passed on and checked by the library)."""
    if not ws.is_cuda or ws.device != device:
        raise ValueError(f"workspace must be a CUDA tensor on {device}")
    if not ws.is_contiguous():
        raise ValueError("workspace must be contiguous")


def _launch(device, stream, fn, *args, owned=()) -> int:
    """Call library entry point `fn` with `device` (the tensors' device) current, passing
    `stream`, or that device's current stream, as the last argument. The library enqueues
    on the current device, so tensors on another GPU would otherwise be read from the
    wrong one.

    `owned` lists the tensors this wrapper allocated (outputs, workspaces). They come from
    torch's caching allocator on the device's current stream; when the kernels run on
    another stream, each is recorded on that stream, so that its memory is not handed out
    again while those kernels may still use it. A stream of another device is refused."""
    import torch
    with torch.cuda.device(device):
        cur = torch.cuda.current_stream(device)
        if stream is None:
            s = cur
        else:
            if torch.device(stream.device) != torch.device(device):
                raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
            s = stream
        status = int(fn(*args, int(s.cuda_stream)))
        if int(s.cuda_stream) != int(cur.cuda_stream):
            for t in owned:
                if t is not None:
                    t.record_stream(s)
        return status


def fwd(q, k, v, causal: bool = False, scale: Optional[float] = None, out=None, lse=None,
        return_lse: bool = True, stream=None) -> Tuple[object, Optional[object]]:
    """O = softmax(scale * Q K^T) V and the per-row natural-log LSE via ``fa_fwd``.

    q [B,Hq,Nq,d], k and v [B,Hkv,Nk,d] (fp16 or bf16, contiguous, same CUDA device).
    Returns (o [B,Hq,Nq,d], lse [B,Hq,Nq] fp32 or None).
    """
    import torch
    _check(q, "q", 4, q.device)
    _check(k, "k", 4, q.device)
    _check(v, "v", 4, q.device)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or dk != d:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    owned = []
    if out is None:
        out = torch.empty_like(q)
        owned.append(out)
    else:
        _check_buf(out, "out", q.shape, q.dtype, q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
        owned.append(lse)
    elif lse is not None:
        _check_buf(lse, "lse", (B, Hq, Nq), torch.float32, q.device)
    st = _launch(q.device, stream, lib().fa_fwd,
                 q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                 lse.data_ptr() if lse is not None else None, B, Hq, Hkv, Nq, Nk, d,
                 1 if causal else 0, float(scale), _dtype_code(q), owned=owned)
    if st != FA_OK:
        raise FAError(st, "fa_fwd")
    return out, lse


def _check_lens(t, name: str, B: int, device) -> None:
    """Per-sequence lengths: int32 [B] on the tensors' device, contiguous (or None)."""
    import torch
    if t is None:
        return
    _check(t, name, 1, device)
    if t.dtype != torch.int32 or t.shape[0] != B:
        raise TypeError(f"{name} must be int32 [B={B}], got {t.dtype} {tuple(t.shape)}")


def fwd_kvcache(q, kcache, vcache, nk: int, causal: bool = True, scale: Optional[float] = None,
                out=None, lse=None, return_lse: bool = True, stream=None, q_lens=None,
                kv_lens=None):
    """Chunked prefill via ``fa_fwd_kvcache``: q [B,Hq,Nq,d] against the first ``nk`` rows of
    kcache, vcache [B,Hkv,cache_len,d] (causal: the chunk is the prefix's last Nq tokens).
    q_lens / kv_lens (int32 [B] on the device, optional) give sequence b its own nq_b <= Nq
    query rows and nk_b <= nk keys; output rows past nq_b are left as they are.
    Returns (o [B,Hq,Nq,d], lse [B,Hq,Nq] fp32 or None).
    """
    import torch
    _check(q, "q", 4, q.device)
    _check(kcache, "kcache", 4, q.device)
    _check(vcache, "vcache", 4, q.device)
    _check_lens(q_lens, "q_lens", q.shape[0], q.device)
    _check_lens(kv_lens, "kv_lens", q.shape[0], q.device)
    if kcache.dtype != q.dtype or vcache.dtype != q.dtype:
        raise TypeError("q, kcache, vcache must share one dtype")
    B, Hq, Nq, d = q.shape
    Bk, Hkv, cache_len, dk = kcache.shape
    if tuple(vcache.shape) != tuple(kcache.shape) or Bk != B or dk != d:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} kcache{tuple(kcache.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    owned = []
    if out is None:
        out = torch.empty_like(q)
        owned.append(out)
    else:
        _check_buf(out, "out", q.shape, q.dtype, q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
        owned.append(lse)
    elif lse is not None:
        _check_buf(lse, "lse", (B, Hq, Nq), torch.float32, q.device)
    st = _launch(q.device, stream, lib().fa_fwd_kvcache,
                 q.data_ptr(), kcache.data_ptr(), vcache.data_ptr(),
                 q_lens.data_ptr() if q_lens is not None else None,
                 kv_lens.data_ptr() if kv_lens is not None else None, out.data_ptr(),
                 lse.data_ptr() if lse is not None else None, B, Hq, Hkv, Nq, int(nk), cache_len, d,
                 1 if causal else 0, float(scale), _dtype_code(q), owned=owned)
    if st != FA_OK:
        raise FAError(st, "fa_fwd_kvcache")
    return out, lse


def _check_pool(q, kpool, vpool, block_table):
    import torch
    _check(kpool, "kpool", 4, q.device)
    _check(vpool, "vpool", 4, q.device)
    _check(block_table, "block_table", 2, q.device)
    if block_table.dtype != torch.int32:
        raise TypeError("block_table must be int32")
    if kpool.dtype != q.dtype or vpool.dtype != q.dtype:
        raise TypeError("q and the page pools must share one dtype")
    if tuple(vpool.shape) != tuple(kpool.shape) or kpool.shape[3] != q.shape[-1]:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} kpool{tuple(kpool.shape)}")
    if block_table.shape[0] != q.shape[0]:
        raise ValueError("block_table needs one row per sequence")


def fwd_paged(q, kpool, vpool, block_table, nk: int, causal: bool = True,
              scale: Optional[float] = None, out=None, lse=None, return_lse: bool = True,
              stream=None, q_lens=None, kv_lens=None):
    """Prefill against a paged KV cache via ``fa_fwd_paged``: q [B,Hq,Nq,d] attends to the
    first ``nk`` tokens of each sequence, kept in pools [num_pages,Hkv,page_size,d] at the
    pages listed by block_table int32 [B, max_pages] (causal: the chunk is the last Nq of
    the nk tokens). q_lens / kv_lens (int32 [B] on the device, optional) give sequence b
    its own nq_b <= Nq query rows and nk_b <= nk tokens; output rows past nq_b are left
    as they are. Returns (o [B,Hq,Nq,d], lse [B,Hq,Nq] fp32 or None).
    """
    import torch
    _check(q, "q", 4, q.device)
    _check_pool(q, kpool, vpool, block_table)
    _check_lens(q_lens, "q_lens", q.shape[0], q.device)
    _check_lens(kv_lens, "kv_lens", q.shape[0], q.device)
    B, Hq, Nq, d = q.shape
    num_pages, Hkv, page_size, _ = kpool.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    owned = []
    if out is None:
        out = torch.empty_like(q)
        owned.append(out)
    else:
        _check_buf(out, "out", q.shape, q.dtype, q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
        owned.append(lse)
    elif lse is not None:
        _check_buf(lse, "lse", (B, Hq, Nq), torch.float32, q.device)
    st = _launch(q.device, stream, lib().fa_fwd_paged,
                 q.data_ptr(), kpool.data_ptr(), vpool.data_ptr(), block_table.data_ptr(),
                 q_lens.data_ptr() if q_lens is not None else None,
                 kv_lens.data_ptr() if kv_lens is not None else None, out.data_ptr(), lse.data_ptr() if lse is not None else None, B, Hq, Hkv, Nq,
                 int(nk), num_pages, page_size, block_table.shape[1], d, 1 if causal else 0,
                 float(scale), _dtype_code(q), owned=owned)
    if st != FA_OK:
        raise FAError(st, "fa_fwd_paged")
    return out, lse


def decode_paged(q, kpool, vpool, block_table, kv_lens, scale: Optional[float] = None, out=None,
                 lse=None, workspace=None, return_lse: bool = True, stream=None):
    """Single-token decode over a paged KV cache via ``fa_decode_paged``.

    q [B,Hq,d]; kpool, vpool [num_pages,Hkv,page_size,d]; block_table int32 [B, max_pages];
    kv_lens int32 [B]; all on the device. Returns (o [B,Hq,d], lse [B,Hq] fp32 or None).
    """
    import torch
    _check(q, "q", 3, q.device)
    _check_pool(q, kpool, vpool, block_table)
    _check(kv_lens, "kv_lens", 1, q.device)
    if kv_lens.dtype != torch.int32 or kv_lens.shape[0] != q.shape[0]:
        raise TypeError("kv_lens must be int32 [B]")
    B, Hq, d = q.shape
    num_pages, Hkv, page_size, _ = kpool.shape
    max_pages = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    owned = []
    if out is None:
        out = torch.empty_like(q)
        owned.append(out)
    else:
        _check_buf(out, "out", q.shape, q.dtype, q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        owned.append(lse)
    elif lse is not None:
        _check_buf(lse, "lse", (B, Hq), torch.float32, q.device)
    if workspace is None:
        workspace = torch.empty(decode_workspace_bytes(B, Hq, max_pages * page_size, d),
                                dtype=torch.uint8, device=q.device)
        owned.append(workspace)
    else:
        _check_workspace(workspace, q.device)
    st = _launch(q.device, stream, lib().fa_decode_paged,
                 q.data_ptr(), kpool.data_ptr(), vpool.data_ptr(), block_table.data_ptr(),
                 kv_lens.data_ptr(), out.data_ptr(), lse.data_ptr() if lse is not None else None, B,
                 Hq, Hkv, num_pages, page_size, max_pages, d, float(scale), _dtype_code(q),
                 workspace.data_ptr(), workspace.numel() * workspace.element_size(), owned=owned)
    if st != FA_OK:
        raise FAError(st, "fa_decode_paged")
    return out, lse


def fwd_fp8(q8, k8, v8, q_descale: float, k_descale: float, v_descale: float,
            causal: bool = False, scale: Optional[float] = None, out=None, lse=None,
            return_lse: bool = True, stream=None):
    """Attention of E4M3 inputs via ``fa_fwd_fp8``: q8 [B,Hq,Nq,128], k8, v8 [B,Hkv,Nk,128]
    as uint8 codes or float8_e4m3fn tensors; the inputs are code x descale per tensor.
    Returns (o [B,Hq,Nq,128] bf16, lse [B,Hq,Nq] fp32 or None)."""
    import torch
    for t, name in ((q8, "q8"), (k8, "k8"), (v8, "v8")):
        _check(t, name, 4, q8.device)
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn):
            raise TypeError(f"{name} must hold E4M3 codes (uint8 or float8_e4m3fn)")
    B, Hq, Nq, d = q8.shape
    Bk, Hkv, Nk, dk = k8.shape
    if tuple(v8.shape) != tuple(k8.shape) or Bk != B or dk != d:
        raise ValueError(f"shape mismatch q{tuple(q8.shape)} k{tuple(k8.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    owned = []
    if out is None:
        out = torch.empty((B, Hq, Nq, d), dtype=torch.bfloat16, device=q8.device)
        owned.append(out)
    else:
        _check_buf(out, "out", (B, Hq, Nq, d), torch.bfloat16, q8.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q8.device)
        owned.append(lse)
    elif lse is not None:
        _check_buf(lse, "lse", (B, Hq, Nq), torch.float32, q8.device)
    st = _launch(q8.device, stream, lib().fa_fwd_fp8,
                 q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), out.data_ptr(),
                 lse.data_ptr() if lse is not None else None, B, Hq, Hkv, Nq, Nk, d,
                 1 if causal else 0, float(scale), float(q_descale), float(k_descale),
                 float(v_descale), owned=owned)
    if st != FA_OK:
        raise FAError(st, "fa_fwd_fp8")
    return out, lse


def bwd_workspace_bytes(B: int, Hq: int, Nq: int) -> int:
    """Scratch bytes ``fa_bwd`` needs for these sizes."""
    return int(lib().fa_bwd_workspace_bytes(B, Hq, Nq))


def bwd(q, k, v, o, lse, dout, causal: bool = False, scale: Optional[float] = None, dq=None,
        dk=None, dv=None, workspace=None, stream=None):
    """Gradients of ``fwd`` via ``fa_bwd``: (dq [B,Hq,Nq,d], dk, dv [B,Hkv,Nk,d]).

    o and lse are ``fwd``'s outputs for q, k, v; dout is the upstream gradient of o.
    """
    import torch
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _check(t, name, 4, q.device)
    if any(t.dtype != q.dtype for t in (k, v, o, dout)):
        raise TypeError("q, k, v, o, dout must share one dtype")
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk_ = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or dk_ != d or tuple(o.shape) != tuple(q.shape) \
            or tuple(dout.shape) != tuple(q.shape):
        raise ValueError("shape mismatch")
    _check_buf(lse, "lse", (B, Hq, Nq), torch.float32, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    for t, name, like in ((dq, "dq", q), (dk, "dk", k), (dv, "dv", v)):
        if t is not None:
            _check_buf(t, name, like.shape, like.dtype, q.device)
    owned = []
    if dq is None:
        dq = torch.empty_like(q)
        owned.append(dq)
    if dk is None:
        dk = torch.empty_like(k)
        owned.append(dk)
    if dv is None:
        dv = torch.empty_like(v)
        owned.append(dv)
    need = bwd_workspace_bytes(B, Hq, Nq)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        owned.append(workspace)
    else:
        _check_workspace(workspace, q.device)
    st = _launch(q.device, stream, lib().fa_bwd,
                 q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                 dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Nq, Nk,
                 d, 1 if causal else 0, float(scale), _dtype_code(q), workspace.data_ptr(),
                 workspace.numel() * workspace.element_size(), owned=owned)
    if st != FA_OK:
        raise FAError(st, "fa_bwd")
    return dq, dk, dv


def decode(q, kcache, vcache, kv_lens, scale: Optional[float] = None, out=None, lse=None,
           workspace=None, return_lse: bool = True, stream=None):
    """Single-token decode over a KV cache via ``fa_decode``.

    q [B,Hq,d]; kcache, vcache [B,Hkv,max_kv_len,d]; kv_lens int32 [B] on the device.
    Returns (o [B,Hq,d], lse [B,Hq] fp32 or None).
    """
    import torch
    _check(q, "q", 3, q.device)
    _check(kcache, "kcache", 4, q.device)
    _check(vcache, "vcache", 4, q.device)
    _check(kv_lens, "kv_lens", 1, q.device)
    if kv_lens.dtype != torch.int32:
        raise TypeError("kv_lens must be int32")
    if kcache.dtype != q.dtype or vcache.dtype != q.dtype:
        raise TypeError("q and the caches must share one dtype")
    B, Hq, d = q.shape
    Bk, Hkv, max_len, dk = kcache.shape
    if tuple(vcache.shape) != tuple(kcache.shape) or Bk != B or dk != d or kv_lens.shape[0] != B:
        raise ValueError("shape mismatch between q, caches and kv_lens")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    owned = []
    if out is None:
        out = torch.empty_like(q)
        owned.append(out)
    else:
        _check_buf(out, "out", q.shape, q.dtype, q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        owned.append(lse)
    elif lse is not None:
        _check_buf(lse, "lse", (B, Hq), torch.float32, q.device)
    need = decode_workspace_bytes(B, Hq, max_len, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        owned.append(workspace)
    else:
        _check_workspace(workspace, q.device)
    st = _launch(q.device, stream, lib().fa_decode,
                 q.data_ptr(), kcache.data_ptr(), vcache.data_ptr(), kv_lens.data_ptr(),
                 out.data_ptr(), lse.data_ptr() if lse is not None else None, B, Hq, Hkv, max_len,
                 d, float(scale), _dtype_code(q), workspace.data_ptr(),
                 workspace.numel() * workspace.element_size(), owned=owned)
    if st != FA_OK:
        raise FAError(st, "fa_decode")
    return out, lse


def decode_noalloc(q, kcache, vcache, kv_lens, scale: Optional[float] = None, out=None, lse=None,
                   return_lse: bool = True, stream=None):
    """Decode via ``fa_decode_noalloc``: same arguments and results as `decode`, but the
    split-KV scratch is the library's own fixed 32 MiB device array, so the library itself
    allocates nothing (for callers that cannot call cudaMalloc: a serving process whose
    device memory is already handed to its own pool, a plugin without an allocator, or a
    latency-critical loop that must avoid cudaMalloc's cost and synchronisation). Calls on
    one device share that scratch: do not let two of them overlap on the GPU. `out` and
    `lse` are allocated here only if the caller does not pass them.
    """
    import torch
    _check(q, "q", 3, q.device)
    _check(kcache, "kcache", 4, q.device)
    _check(vcache, "vcache", 4, q.device)
    _check(kv_lens, "kv_lens", 1, q.device)
    if kv_lens.dtype != torch.int32:
        raise TypeError("kv_lens must be int32")
    if kcache.dtype != q.dtype or vcache.dtype != q.dtype:
        raise TypeError("q and the caches must share one dtype")
    B, Hq, d = q.shape
    Bk, Hkv, max_len, dk = kcache.shape
    if tuple(vcache.shape) != tuple(kcache.shape) or Bk != B or dk != d or kv_lens.shape[0] != B:
        raise ValueError("shape mismatch between q, caches and kv_lens")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    owned = []
    if out is None:
        out = torch.empty_like(q)
        owned.append(out)
    else:
        _check_buf(out, "out", q.shape, q.dtype, q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        owned.append(lse)
    elif lse is not None:
        _check_buf(lse, "lse", (B, Hq), torch.float32, q.device)
    st = _launch(q.device, stream, lib().fa_decode_noalloc,
                 q.data_ptr(), kcache.data_ptr(), vcache.data_ptr(), kv_lens.data_ptr(),
                 out.data_ptr(), lse.data_ptr() if lse is not None else None, B, Hq, Hkv, max_len,
                 d, float(scale), _dtype_code(q), owned=owned)
    if st != FA_OK:
        raise FAError(st, "fa_decode_noalloc")
    return out, lse
