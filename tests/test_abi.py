"""CPU checks of the C-ABI library: it loads, exports every symbol the header declares,
and rejects bad arguments on the host before touching CUDA (no GPU needed)."""
import ctypes
import os
import re

import pytest

import io_aware_exact_28_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


def header_functions():
    with open(HEADER) as f:
        src = f.read()
    return re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", src)


def test_library_loads_and_targets_sm100a():
    assert os.path.exists(fa.LIB_PATH)
    assert "sm_100a" in fa.build_info()


def test_every_declared_symbol_is_exported():
    names = header_functions()
    assert set(names) == set(fa.EXPORTED_SYMBOLS), names
    L = ctypes.CDLL(fa.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings():
    for code in range(7):
        assert fa.status_string(code).startswith("FA_")
    assert fa.status_string(99) == "FA_ERR_UNKNOWN"


def _fwd(L, q=16, k=16, v=16, o=16, lse=None, B=1, Hq=2, Hkv=1, Nq=128, Nk=128, d=64, causal=1,
         scale=0.125, dtype=0):
    return L.fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, dtype, None)


def test_fwd_rejects_bad_arguments_without_cuda():
    L = fa.lib()
    assert _fwd(L, q=None) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, o=None) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, B=0) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, Nq=0) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, Nk=-3) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, Hq=3, Hkv=2) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, causal=2) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, scale=float("inf")) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, scale=float("nan")) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, scale=-1.0) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, d=96) == fa.FA_ERR_UNSUPPORTED
    assert _fwd(L, dtype=7) == fa.FA_ERR_UNSUPPORTED
    assert _fwd(L, q=24) == fa.FA_ERR_ALIGNMENT
    assert _fwd(L, lse=18) == fa.FA_ERR_ALIGNMENT


def test_fwd_kvcache_rejects_bad_arguments_without_cuda():
    L = fa.lib()

    def call(Nk=128, cache_len=256, **kw):
        a = dict(q=16, k=16, v=16, o=16, lse=None, B=1, Hq=2, Hkv=1, Nq=64, d=64, causal=1,
                 scale=0.125, dtype=0)
        a.update(kw)
        return L.fa_fwd_kvcache(a["q"], a["k"], a["v"], a.get("q_lens"), a.get("kv_lens"), a["o"],
                                a["lse"], a["B"], a["Hq"], a["Hkv"], a["Nq"], Nk, cache_len, a["d"],
                                a["causal"], a["scale"], a["dtype"], None)
    assert call(Nk=257, cache_len=256) == fa.FA_ERR_INVALID_ARG    # prefix longer than the cache
    assert call(cache_len=0) == fa.FA_ERR_INVALID_ARG
    assert call(Nk=0) == fa.FA_ERR_INVALID_ARG
    assert call(q=None) == fa.FA_ERR_INVALID_ARG
    assert call(d=96) == fa.FA_ERR_UNSUPPORTED
    assert call(k=24) == fa.FA_ERR_ALIGNMENT
    assert call(q_lens=18) == fa.FA_ERR_ALIGNMENT        # per-sequence lengths: 4-byte aligned
    assert call(kv_lens=34) == fa.FA_ERR_ALIGNMENT


def test_bwd_rejects_bad_arguments_without_cuda():
    L = fa.lib()
    ws_need = L.fa_bwd_workspace_bytes(1, 2, 200)
    assert ws_need == 2 * 2 * 256 * 4          # L*log2(e) and D, each [B*Hq, Nq padded to 256]
    assert L.fa_bwd_workspace_bytes(0, 2, 200) == 0

    def call(**kw):
        a = dict(q=16, k=16, v=16, o=16, lse=16, do=16, dq=16, dk=16, dv=16, B=1, Hq=2, Hkv=1,
                 Nq=200, Nk=200, d=64, causal=1, scale=0.125, dtype=0, ws=16, ws_bytes=ws_need)
        a.update(kw)
        return L.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["do"], a["dq"], a["dk"], a["dv"],
                        a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"], a["d"], a["causal"], a["scale"],
                        a["dtype"], a["ws"], a["ws_bytes"], None)
    assert call(lse=None) == fa.FA_ERR_INVALID_ARG
    assert call(dv=None) == fa.FA_ERR_INVALID_ARG
    assert call(Nk=0) == fa.FA_ERR_INVALID_ARG
    assert call(Hq=3, Hkv=2) == fa.FA_ERR_INVALID_ARG
    assert call(d=80) == fa.FA_ERR_UNSUPPORTED
    assert call(dk=8) == fa.FA_ERR_ALIGNMENT
    assert call(ws_bytes=ws_need - 1) == fa.FA_ERR_WORKSPACE
    assert call(ws=None) == fa.FA_ERR_WORKSPACE


def test_decode_rejects_bad_arguments_without_cuda():
    L = fa.lib()
    need = fa.decode_workspace_bytes(2, 8, 4096, 128)

    def call(q=16, kc=16, vc=16, lens=16, o=16, lse=None, B=2, Hq=8, Hkv=2, max_len=4096, d=128,
             scale=0.088, dtype=1, ws=32, ws_bytes=need):
        return L.fa_decode(q, kc, vc, lens, o, lse, B, Hq, Hkv, max_len, d, scale, dtype, ws,
                           ws_bytes, None)
    assert call(lens=None) == fa.FA_ERR_INVALID_ARG
    assert call(max_len=0) == fa.FA_ERR_INVALID_ARG
    assert call(Hq=6, Hkv=4) == fa.FA_ERR_INVALID_ARG
    assert call(d=80) == fa.FA_ERR_UNSUPPORTED
    assert call(kc=8) == fa.FA_ERR_ALIGNMENT
    assert call(ws=None) == fa.FA_ERR_WORKSPACE
    assert call(ws_bytes=need - 1) == fa.FA_ERR_WORKSPACE


def test_workspace_size_covers_every_split():
    # one fp32 row of d plus one fp32 LSE per (sequence, head, split), 256-byte aligned parts
    for (B, Hq, max_len, d) in [(64, 32, 4096, 128), (1, 1, 1, 64), (3, 8, 1000, 128)]:
        n = fa.decode_workspace_bytes(B, Hq, max_len, d)
        assert n >= B * Hq * (d + 1) * 4
        assert n % 256 == 0
    assert fa.decode_workspace_bytes(0, 8, 128, 64) == 0


def test_paged_entry_points_reject_bad_arguments_without_cuda():
    L = fa.lib()
    need = fa.decode_workspace_bytes(2, 8, 16 * 64, 128)

    def dec(q=16, kp=16, vp=16, table=16, lens=16, o=16, B=2, Hq=8, Hkv=2, num_pages=40,
            page_size=64, max_pages=16, d=128, ws=32, ws_bytes=need):
        return L.fa_decode_paged(q, kp, vp, table, lens, o, None, B, Hq, Hkv, num_pages, page_size,
                                 max_pages, d, 0.088, 1, ws, ws_bytes, None)

    def fwd(q=16, kp=16, vp=16, table=16, o=16, Nq=64, Nk=300, num_pages=40, page_size=32,
            max_pages=10, d=64):
        return L.fa_fwd_paged(q, kp, vp, table, None, None, o, None, 1, 2, 1, Nq, Nk, num_pages,
                              page_size, max_pages, d, 1, 0.125, 0, None)
    for call in (dec, fwd):
        assert call(table=None) == fa.FA_ERR_INVALID_ARG
        assert call(num_pages=0) == fa.FA_ERR_INVALID_ARG
        assert call(max_pages=0) == fa.FA_ERR_INVALID_ARG
        assert call(page_size=48) == fa.FA_ERR_UNSUPPORTED     # not a power of two
        assert call(page_size=8) == fa.FA_ERR_UNSUPPORTED      # below 16 rows
        assert call(table=18) == fa.FA_ERR_ALIGNMENT
        assert call(kp=24) == fa.FA_ERR_ALIGNMENT
        assert call(num_pages=2**31 - 1) == fa.FA_ERR_INVALID_ARG   # past-the-pool index overflows
        assert call(d=96) == fa.FA_ERR_UNSUPPORTED
    assert fwd(Nk=321) == fa.FA_ERR_INVALID_ARG                 # more tokens than the table covers
    assert dec(ws_bytes=need - 1) == fa.FA_ERR_WORKSPACE
    assert dec(max_pages=1 << 26) == fa.FA_ERR_INVALID_ARG      # max_pages * page_size >= 2^31


def test_fwd_fp8_rejects_bad_arguments_without_cuda():
    L = fa.lib()

    def call(q=16, k=16, v=16, o=16, lse=None, B=1, Hq=2, Hkv=1, Nq=128, Nk=128, d=128, causal=1,
             scale=0.088, dq=0.01, dk=0.01, dv=0.01):
        return L.fa_fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, dq, dk, dv, None)
    assert call(q=None) == fa.FA_ERR_INVALID_ARG
    assert call(Nk=0) == fa.FA_ERR_INVALID_ARG
    assert call(Hq=3, Hkv=2) == fa.FA_ERR_INVALID_ARG
    assert call(dq=0.0) == fa.FA_ERR_INVALID_ARG
    assert call(dv=float("nan")) == fa.FA_ERR_INVALID_ARG
    assert call(dk=-1.0) == fa.FA_ERR_INVALID_ARG
    assert call(d=64) == fa.FA_ERR_UNSUPPORTED        # d = 128 only
    assert call(v=40) == fa.FA_ERR_ALIGNMENT


def test_every_declaration_states_its_source():
    """Each FA_API declaration sits under a comment block that cites the page passage
    defining the operation, or says it is not an operation of the pages."""
    import re
    with open(os.path.join(ROOT, "include", "fa.h"), encoding="utf-8") as f:
        src = f.read()
    names = []
    for m in re.finditer(r"FA_API\s+[^;]*?\b(fa_\w+)\s*\(", src):
        before = src[:m.start()]
        block = before[before.rfind("/*"):]
        assert "*/" in block, m.group(1)
        block = re.sub(r"\s*\n\s*\*(?!/)\s*", " ", block)     # one line, no leading stars
        low = block.lower()
        assert 'page "' in block or "not an operation of the pages" in low or \
            "not operations of the pages" in low or "not from the pages" in low or \
            "not on the pages" in low, m.group(1)
        names.append(m.group(1))
    assert len(names) >= 15
