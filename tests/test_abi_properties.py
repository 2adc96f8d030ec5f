"""Property tests of the C ABI's host-side argument checks (CPU, no GPU needed).

Each example starts from an argument set that passes every check and then breaks it in
exactly one way, drawn at random from one class of fault:

- a required pointer is null, a size or count is out of range, the query/KV head counts
  do not divide, the scale is not a finite positive number, or a product of sizes
  overflows the kernels' 32-bit indexing: FA_ERR_INVALID_ARG;
- the head dimension or dtype is not supported: FA_ERR_UNSUPPORTED;
- a pointer is misaligned (16 bytes for tensors, 4 for int32 / fp32 vectors):
  FA_ERR_ALIGNMENT;
- (decode, backward) the workspace is missing or smaller than fa_decode_workspace_bytes
  or fa_bwd_workspace_bytes says: FA_ERR_WORKSPACE;
- (chunked prefill) the cache is shorter than the keys used: FA_ERR_INVALID_ARG;
- (paged pool) no table, a page or table count <= 0, pool or table index overflow, or a
  table too short for the keys: FA_ERR_INVALID_ARG; a page size that is not a power of two
  or is below 16: FA_ERR_UNSUPPORTED;
- (E4M3) a descale that is not finite and positive: FA_ERR_INVALID_ARG; d other than 128:
  FA_ERR_UNSUPPORTED.

The call must return exactly that status. Every example carries a fault, so no example
reaches a kernel launch; the pointers are never dereferenced.
"""
import math

from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import io_aware_exact_28_b200 as fa

SETTINGS = settings(derandomize=True, max_examples=300, deadline=None,
                    suppress_health_check=[HealthCheck.too_slow])

aligned = st.integers(1, 1 << 24).map(lambda i: 16 * i)          # 16-byte aligned addresses
misaligned = st.tuples(st.integers(1, 1 << 24), st.integers(1, 15)).map(lambda t: 16 * t[0] + t[1])


@st.composite
def valid_fwd(draw):
    Hkv = draw(st.integers(1, 16))
    g = draw(st.integers(1, 8))
    return dict(q=draw(aligned), k=draw(aligned), v=draw(aligned), o=draw(aligned),
                lse=draw(st.one_of(st.none(), st.integers(1, 1 << 24).map(lambda i: 4 * i))),
                B=draw(st.integers(1, 256)), Hq=Hkv * g, Hkv=Hkv,
                Nq=draw(st.integers(1, 1 << 20)), Nk=draw(st.integers(1, 1 << 20)),
                d=draw(st.sampled_from([64, 128])), causal=draw(st.sampled_from([0, 1])),
                scale=draw(st.floats(1e-3, 10.0)), dtype=draw(st.sampled_from([0, 1])))


def call_fwd(a):
    return fa.lib().fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                           a["Nq"], a["Nk"], a["d"], a["causal"], a["scale"], a["dtype"], None)


@st.composite
def invalid_arg_fault(draw, a):
    kind = draw(st.sampled_from(["null", "B", "Hq", "Hkv", "ratio", "Nq", "Nk", "causal",
                                 "scale", "overflow"]))
    a = dict(a)
    if kind == "null":
        a[draw(st.sampled_from(["q", "k", "v", "o"]))] = None
    elif kind in ("B", "Nq", "Nk"):
        a[kind] = draw(st.integers(-(1 << 31), 0))
    elif kind == "Hq":
        a["Hq"] = draw(st.integers(-(1 << 31), 0))
    elif kind == "Hkv":
        a["Hkv"] = draw(st.integers(-(1 << 31), 0))
    elif kind == "ratio":
        Hkv = draw(st.integers(2, 16))
        a["Hkv"], a["Hq"] = Hkv, Hkv * draw(st.integers(1, 8)) + draw(st.integers(1, Hkv - 1))
    elif kind == "causal":
        a["causal"] = draw(st.one_of(st.integers(2, 1 << 20), st.integers(-(1 << 20), -1)))
    elif kind == "scale":
        a["scale"] = draw(st.sampled_from([math.nan, math.inf, -math.inf, 0.0, -0.5, -1e30]))
    else:                                   # B * Hq reaches 2^31 query heads
        a["Hkv"] = 1
        a["Hq"] = draw(st.integers(2, 64))
        a["B"] = -(-(1 << 31) // a["Hq"]) + draw(st.integers(0, 64))   # ceil(2^31 / Hq) + k
        assert a["B"] * a["Hq"] >= (1 << 31)
    return a


@SETTINGS
@given(st.data())
def test_fwd_invalid_arguments(data):
    a = data.draw(invalid_arg_fault(data.draw(valid_fwd())))
    assert call_fwd(a) == fa.FA_ERR_INVALID_ARG, a


@SETTINGS
@given(valid_fwd(), st.data())
def test_fwd_unsupported(a, data):
    if data.draw(st.booleans()):
        a["d"] = data.draw(st.integers(-8, 512).filter(lambda d: d not in (64, 128)))
    else:
        a["dtype"] = data.draw(st.integers(-4, 64).filter(lambda t: t not in (0, 1)))
    assert call_fwd(a) == fa.FA_ERR_UNSUPPORTED, a


@SETTINGS
@given(valid_fwd(), st.data())
def test_fwd_misaligned(a, data):
    which = data.draw(st.sampled_from(["q", "k", "v", "o", "lse"]))
    if which == "lse":
        a["lse"] = data.draw(st.tuples(st.integers(1, 1 << 24), st.integers(1, 3))
                             .map(lambda t: 4 * t[0] + t[1]))
    else:
        a[which] = data.draw(misaligned)
    assert call_fwd(a) == fa.FA_ERR_ALIGNMENT, a


@st.composite
def valid_decode(draw):
    Hkv = draw(st.integers(1, 16))
    a = dict(q=draw(aligned), kc=draw(aligned), vc=draw(aligned),
             lens=draw(st.integers(1, 1 << 24).map(lambda i: 4 * i)), o=draw(aligned),
             lse=draw(st.one_of(st.none(), st.integers(1, 1 << 24).map(lambda i: 4 * i))),
             B=draw(st.integers(1, 512)), Hkv=Hkv, Hq=Hkv * draw(st.integers(1, 8)),
             max_len=draw(st.integers(1, 1 << 17)), d=draw(st.sampled_from([64, 128])),
             scale=draw(st.floats(1e-3, 10.0)), dtype=draw(st.sampled_from([0, 1])),
             ws=draw(aligned))
    a["ws_bytes"] = fa.decode_workspace_bytes(a["B"], a["Hq"], a["max_len"], a["d"])
    return a


def call_decode(a):
    return fa.lib().fa_decode(a["q"], a["kc"], a["vc"], a["lens"], a["o"], a["lse"], a["B"],
                              a["Hq"], a["Hkv"], a["max_len"], a["d"], a["scale"], a["dtype"],
                              a["ws"], a["ws_bytes"], None)


@SETTINGS
@given(valid_decode(), st.data())
def test_decode_single_faults(a, data):
    kind = data.draw(st.sampled_from(["null", "max_len", "B", "ratio", "scale", "unsupported",
                                      "misaligned", "lens_misaligned", "no_workspace",
                                      "small_workspace"]))
    if kind == "null":
        a[data.draw(st.sampled_from(["q", "kc", "vc", "lens", "o"]))] = None
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "max_len":
        a["max_len"] = data.draw(st.integers(-(1 << 31), 0))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "B":
        a["B"] = data.draw(st.one_of(st.integers(-(1 << 31), 0), st.integers(65536, 1 << 30)))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "ratio":
        Hkv = data.draw(st.integers(2, 16))
        a["Hkv"], a["Hq"] = Hkv, Hkv * data.draw(st.integers(1, 8)) + data.draw(st.integers(1, Hkv - 1))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "scale":
        a["scale"] = data.draw(st.sampled_from([math.nan, math.inf, 0.0, -2.0]))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "unsupported":
        a["d"] = data.draw(st.integers(1, 512).filter(lambda d: d not in (64, 128)))
        want = fa.FA_ERR_UNSUPPORTED
    elif kind == "misaligned":
        a[data.draw(st.sampled_from(["q", "kc", "vc", "o"]))] = data.draw(misaligned)
        want = fa.FA_ERR_ALIGNMENT
    elif kind == "lens_misaligned":
        a["lens"] = 4 * data.draw(st.integers(1, 1 << 24)) + data.draw(st.integers(1, 3))
        want = fa.FA_ERR_ALIGNMENT
    elif kind == "no_workspace":
        a["ws"] = None
        want = fa.FA_ERR_WORKSPACE
    else:
        a["ws_bytes"] = data.draw(st.integers(0, a["ws_bytes"] - 1))
        want = fa.FA_ERR_WORKSPACE
    assert call_decode(a) == want, (kind, a)


# ---- fa_bwd -------------------------------------------------------------------------

@st.composite
def valid_bwd(draw):
    Hkv = draw(st.integers(1, 16))
    a = dict(q=draw(aligned), k=draw(aligned), v=draw(aligned), o=draw(aligned),
             lse=draw(st.integers(1, 1 << 24).map(lambda i: 4 * i)), do=draw(aligned),
             dq=draw(aligned), dk=draw(aligned), dv=draw(aligned),
             B=draw(st.integers(1, 64)), Hq=Hkv * draw(st.integers(1, 8)), Hkv=Hkv,
             Nq=draw(st.integers(1, 4096)), Nk=draw(st.integers(1, 1 << 20)),
             d=draw(st.sampled_from([64, 128])), causal=draw(st.sampled_from([0, 1])),
             scale=draw(st.floats(1e-3, 10.0)), dtype=draw(st.sampled_from([0, 1])),
             ws=draw(aligned))
    a["ws_bytes"] = fa.lib().fa_bwd_workspace_bytes(a["B"], a["Hq"], a["Nq"])
    return a


def call_bwd(a):
    return fa.lib().fa_bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["do"], a["dq"], a["dk"],
                           a["dv"], a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"], a["d"],
                           a["causal"], a["scale"], a["dtype"], a["ws"], a["ws_bytes"], None)


BWD_TENSORS = ["q", "k", "v", "o", "do", "dq", "dk", "dv"]


@SETTINGS
@given(valid_bwd(), st.data())
def test_bwd_single_faults(a, data):
    """Every tensor pointer, the LSE included, is required; the grid limits are B * Hq and
    B * Hkv below 65536 and B * Hq * (Nq rounded up to 128) * 32 below 2^31."""
    kind = data.draw(st.sampled_from(["null", "size", "ratio", "causal", "scale", "heads",
                                      "rows", "unsupported", "misaligned", "lse_misaligned",
                                      "ws_misaligned", "no_workspace", "small_workspace"]))
    if kind == "null":
        a[data.draw(st.sampled_from(BWD_TENSORS + ["lse"]))] = None
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "size":
        a[data.draw(st.sampled_from(["B", "Hq", "Hkv", "Nq", "Nk"]))] = data.draw(st.integers(-(1 << 31), 0))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "ratio":
        Hkv = data.draw(st.integers(2, 16))
        a["Hkv"], a["Hq"] = Hkv, Hkv * data.draw(st.integers(1, 8)) + data.draw(st.integers(1, Hkv - 1))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "causal":
        a["causal"] = data.draw(st.one_of(st.integers(2, 1 << 20), st.integers(-(1 << 20), -1)))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "scale":
        a["scale"] = data.draw(st.sampled_from([math.nan, math.inf, -math.inf, 0.0, -0.5]))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "heads":                   # B * Hq reaches 65536 (one KV head)
        a["Hkv"] = 1
        a["Hq"] = data.draw(st.integers(1, 64))
        a["B"] = -(-65536 // a["Hq"]) + data.draw(st.integers(0, 64))
        a["Nq"] = 1
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "rows":                    # B * Hq * padded Nq * 32 reaches 2^31
        a["Nq"] = -(-(1 << 26) // (a["B"] * a["Hq"])) + data.draw(st.integers(0, 1 << 12))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "unsupported":
        if data.draw(st.booleans()):
            a["d"] = data.draw(st.integers(-8, 512).filter(lambda d: d not in (64, 128)))
        else:
            a["dtype"] = data.draw(st.integers(-4, 64).filter(lambda t: t not in (0, 1)))
        want = fa.FA_ERR_UNSUPPORTED
    elif kind == "misaligned":
        a[data.draw(st.sampled_from(BWD_TENSORS))] = data.draw(misaligned)
        want = fa.FA_ERR_ALIGNMENT
    elif kind == "lse_misaligned":
        a["lse"] = 4 * data.draw(st.integers(1, 1 << 24)) + data.draw(st.integers(1, 3))
        want = fa.FA_ERR_ALIGNMENT
    elif kind == "ws_misaligned":
        a["ws"] = data.draw(misaligned)
        want = fa.FA_ERR_ALIGNMENT
    elif kind == "no_workspace":
        a["ws"] = None
        want = fa.FA_ERR_WORKSPACE
    else:
        a["ws_bytes"] = data.draw(st.integers(0, a["ws_bytes"] - 1))
        want = fa.FA_ERR_WORKSPACE
    assert call_bwd(a) == want, (kind, a)


# ---- fa_fwd_kvcache, fa_fwd_paged, fa_fwd_fp8 ---------------------------------------

def call_kvcache(a):
    return fa.lib().fa_fwd_kvcache(a["q"], a["k"], a["v"], a["q_lens"], a["kv_lens"], a["o"],
                                   a["lse"], a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"],
                                   a["cache_len"], a["d"], a["causal"], a["scale"], a["dtype"], None)


@st.composite
def valid_kvcache(draw):
    a = draw(valid_fwd())
    a["cache_len"] = a["Nk"] + draw(st.integers(0, 1 << 20))
    a["q_lens"] = draw(st.one_of(st.none(), st.integers(1, 1 << 24).map(lambda i: 4 * i)))
    a["kv_lens"] = draw(st.one_of(st.none(), st.integers(1, 1 << 24).map(lambda i: 4 * i)))
    return a


@SETTINGS
@given(valid_kvcache(), st.data())
def test_fwd_kvcache_single_faults(a, data):
    """fa_fwd's faults, plus a cache shorter than the keys used and misaligned length
    vectors."""
    kind = data.draw(st.sampled_from(["fwd", "short_cache", "no_cache", "lens_misaligned"]))
    if kind == "fwd":
        a = data.draw(invalid_arg_fault(a))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "short_cache":
        a["Nk"] = max(a["Nk"], 2)
        a["cache_len"] = data.draw(st.integers(1, a["Nk"] - 1))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "no_cache":
        a["cache_len"] = data.draw(st.integers(-(1 << 31), 0))
        want = fa.FA_ERR_INVALID_ARG
    else:
        a[data.draw(st.sampled_from(["q_lens", "kv_lens"]))] = \
            4 * data.draw(st.integers(1, 1 << 24)) + data.draw(st.integers(1, 3))
        want = fa.FA_ERR_ALIGNMENT
    assert call_kvcache(a) == want, (kind, a)


@st.composite
def valid_paged_fwd(draw):
    a = draw(valid_fwd())
    a["Nk"] = draw(st.integers(1, 1 << 16))
    a["page_size"] = 1 << draw(st.integers(4, 10))
    a["max_pages"] = -(-a["Nk"] // a["page_size"]) + draw(st.integers(0, 64))
    a["num_pages"] = draw(st.integers(1, (1 << 24) // a["Hkv"]))
    a["table"] = 4 * draw(st.integers(1, 1 << 24))
    a["q_lens"] = draw(st.one_of(st.none(), st.integers(1, 1 << 24).map(lambda i: 4 * i)))
    a["kv_lens"] = draw(st.one_of(st.none(), st.integers(1, 1 << 24).map(lambda i: 4 * i)))
    return a


def call_paged_fwd(a):
    return fa.lib().fa_fwd_paged(a["q"], a["k"], a["v"], a["table"], a["q_lens"], a["kv_lens"],
                                 a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"],
                                 a["num_pages"], a["page_size"], a["max_pages"], a["d"], a["causal"],
                                 a["scale"], a["dtype"], None)


@st.composite
def paged_fault(draw, a):
    """One fault of the page pool's description: (argument changes, expected status)."""
    a = dict(a)
    kind = draw(st.sampled_from(["no_table", "num_pages", "max_pages", "page_size_neg",
                                 "page_size_odd", "page_size_small", "pool_overflow",
                                 "table_overflow", "table_misaligned"]))
    if kind == "no_table":
        a["table"] = None
        want = fa.FA_ERR_INVALID_ARG
    elif kind in ("num_pages", "max_pages"):
        a[kind] = draw(st.integers(-(1 << 31), 0))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "page_size_neg":
        a["page_size"] = draw(st.integers(-(1 << 31), 0))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "page_size_odd":           # not a power of two (max_pages keeps up with Nk)
        a["page_size"] = draw(st.integers(17, 1 << 10).filter(lambda p: p & (p - 1)))
        a["max_pages"] = -(-a["Nk"] // a["page_size"]) + 1
        want = fa.FA_ERR_UNSUPPORTED
    elif kind == "page_size_small":
        a["page_size"] = draw(st.sampled_from([1, 2, 4, 8]))
        a["max_pages"] = -(-a["Nk"] // a["page_size"])
        want = fa.FA_ERR_UNSUPPORTED
    elif kind == "pool_overflow":           # num_pages * Hkv reaches 2^31 - 1
        a["num_pages"] = -(-((1 << 31) - 1) // a["Hkv"]) + draw(st.integers(0, 64))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "table_overflow":          # max_pages * page_size reaches 2^31
        a["max_pages"] = ((1 << 31) // a["page_size"]) + draw(st.integers(0, 64))
        want = fa.FA_ERR_INVALID_ARG
    else:
        a["table"] = 4 * draw(st.integers(1, 1 << 24)) + draw(st.integers(1, 3))
        want = fa.FA_ERR_ALIGNMENT
    return a, want, kind


@SETTINGS
@given(valid_paged_fwd(), st.data())
def test_fwd_paged_single_faults(a, data):
    """fa_fwd's faults, the pool's, and a table too short for the keys used."""
    kind = data.draw(st.sampled_from(["fwd", "pool", "short_table"]))
    if kind == "fwd":
        a = data.draw(invalid_arg_fault(a))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "pool":
        a, want, kind = data.draw(paged_fault(a))
    else:
        a["Nk"] = max(a["Nk"], a["page_size"] + 1)
        a["max_pages"] = data.draw(st.integers(1, (a["Nk"] - 1) // a["page_size"]))
        want = fa.FA_ERR_INVALID_ARG
    assert call_paged_fwd(a) == want, (kind, a)


@st.composite
def valid_paged_decode(draw):
    Hkv = draw(st.integers(1, 16))
    a = dict(q=draw(aligned), k=draw(aligned), v=draw(aligned),
             lens=draw(st.integers(1, 1 << 24).map(lambda i: 4 * i)), o=draw(aligned),
             lse=draw(st.one_of(st.none(), st.integers(1, 1 << 24).map(lambda i: 4 * i))),
             B=draw(st.integers(1, 512)), Hkv=Hkv, Hq=Hkv * draw(st.integers(1, 8)),
             page_size=1 << draw(st.integers(4, 10)), max_pages=draw(st.integers(1, 256)),
             d=draw(st.sampled_from([64, 128])), scale=draw(st.floats(1e-3, 10.0)),
             dtype=draw(st.sampled_from([0, 1])), ws=draw(aligned),
             table=4 * draw(st.integers(1, 1 << 24)))
    a["Nk"] = a["page_size"] * a["max_pages"]
    a["num_pages"] = draw(st.integers(1, (1 << 24) // Hkv))
    a["ws_bytes"] = fa.decode_workspace_bytes(a["B"], a["Hq"], a["Nk"], a["d"])
    return a


def call_paged_decode(a):
    return fa.lib().fa_decode_paged(a["q"], a["k"], a["v"], a["table"], a["lens"], a["o"], a["lse"],
                                    a["B"], a["Hq"], a["Hkv"], a["num_pages"], a["page_size"],
                                    a["max_pages"], a["d"], a["scale"], a["dtype"], a["ws"],
                                    a["ws_bytes"], None)


@SETTINGS
@given(valid_paged_decode(), st.data())
def test_decode_paged_single_faults(a, data):
    """The pool's faults, and fa_decode's own: null or misaligned tensors, the workspace."""
    kind = data.draw(st.sampled_from(["pool", "null", "misaligned", "no_workspace",
                                      "small_workspace", "unsupported"]))
    if kind == "pool":
        a, want, kind = data.draw(paged_fault(a))
    elif kind == "null":
        a[data.draw(st.sampled_from(["q", "k", "v", "lens", "o"]))] = None
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "misaligned":
        a[data.draw(st.sampled_from(["q", "k", "v", "o"]))] = data.draw(misaligned)
        want = fa.FA_ERR_ALIGNMENT
    elif kind == "no_workspace":
        a["ws"] = None
        want = fa.FA_ERR_WORKSPACE
    elif kind == "small_workspace":
        a["ws_bytes"] = data.draw(st.integers(0, a["ws_bytes"] - 1))
        want = fa.FA_ERR_WORKSPACE
    else:
        a["d"] = data.draw(st.integers(1, 512).filter(lambda d: d not in (64, 128)))
        want = fa.FA_ERR_UNSUPPORTED
    assert call_paged_decode(a) == want, (kind, a)


@st.composite
def valid_fp8(draw):
    a = draw(valid_fwd())
    a["d"] = 128
    for key in ("dq", "dk", "dv"):
        a[key] = draw(st.floats(1e-6, 1e3))
    return a


def call_fp8(a):
    return fa.lib().fa_fwd_fp8(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                               a["Nq"], a["Nk"], a["d"], a["causal"], a["scale"], a["dq"], a["dk"],
                               a["dv"], None)


@SETTINGS
@given(valid_fp8(), st.data())
def test_fwd_fp8_single_faults(a, data):
    """fa_fwd's faults, a descale that is not finite and positive, d other than 128, and
    misaligned tensors."""
    kind = data.draw(st.sampled_from(["fwd", "descale", "d", "misaligned"]))
    if kind == "fwd":
        a = data.draw(invalid_arg_fault(a))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "descale":
        a[data.draw(st.sampled_from(["dq", "dk", "dv"]))] = \
            data.draw(st.sampled_from([math.nan, math.inf, -math.inf, 0.0, -1.0, -1e-30]))
        want = fa.FA_ERR_INVALID_ARG
    elif kind == "d":
        a["d"] = data.draw(st.integers(-8, 512).filter(lambda d: d != 128))
        want = fa.FA_ERR_UNSUPPORTED
    else:
        a[data.draw(st.sampled_from(["q", "k", "v", "o"]))] = data.draw(misaligned)
        want = fa.FA_ERR_ALIGNMENT
    assert call_fp8(a) == want, (kind, a)
