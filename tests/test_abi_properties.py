"""Property tests of the C ABI's host-side argument checks (CPU, no GPU needed).

Each example starts from an argument set that passes every check and then breaks it in
exactly one way, drawn at random from one class of fault:

- a required pointer is null, a size or count is out of range, the query/KV head counts
  do not divide, the scale is not a finite positive number, or a product of sizes
  overflows the kernels' 32-bit indexing: FA_ERR_INVALID_ARG;
- the head dimension or dtype is not supported: FA_ERR_UNSUPPORTED;
- a pointer is misaligned (16 bytes for tensors, 4 for int32 / fp32 vectors):
  FA_ERR_ALIGNMENT;
- (decode) the workspace is missing or smaller than fa_decode_workspace_bytes says:
  FA_ERR_WORKSPACE.

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
