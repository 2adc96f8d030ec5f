"""Static checks that every device-side wait in the CUDA sources is bounded (CPU only).

* The mbarrier poll instruction appears once, in `mbar_try_wait` (csrc/sm100.cuh).
* `mbar_try_wait` is called only inside `mbar_wait` (which gives up after the wait
  limit or when the CTA's abort flag is raised, recording FA_ERR_DEVICE_TIMEOUT) and
  inside `mbar_wait_drain` (a fixed limit, for the abort path). Both read the global
  timer inside their loop.
* No device code stops a kernel by trapping or by a device-side assert: errors are status
  words the host reads.
"""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "io_aware_exact_28_b200", "csrc")


def _sources():
    out = {}
    for n in sorted(os.listdir(CSRC)):
        if n.endswith((".cu", ".cuh")):
            with open(os.path.join(CSRC, n), encoding="utf-8") as f:
                out[n] = f.read()
    assert "sm100.cuh" in out and len(out) >= 5
    return out


def _function_body(src, name):
    """Text of the body of the (first) function `name` defined in src."""
    m = re.search(r"\b" + re.escape(name) + r"\s*\([^;{]*\)\s*\{", src)
    assert m, name
    depth, i = 0, m.end() - 1
    while True:
        if src[i] == "{":
            depth += 1
        elif src[i] == "}":
            depth -= 1
            if depth == 0:
                return src[m.start():i + 1]
        i += 1


def test_the_poll_instruction_lives_in_one_helper():
    srcs = _sources()
    hits = [(n, m.start()) for n, s in srcs.items() for m in re.finditer(r"mbarrier\.try_wait", s)]
    assert len(hits) == 1 and hits[0][0] == "sm100.cuh", hits
    assert "mbarrier.try_wait" in _function_body(srcs["sm100.cuh"], "mbar_try_wait")


def test_polls_happen_only_inside_the_bounded_waits():
    srcs = _sources()
    sm = srcs["sm100.cuh"]
    allowed = [_function_body(sm, "mbar_wait"), _function_body(sm, "mbar_wait_drain")]
    for body in allowed:            # the loop compares elapsed global time with a limit
        assert re.search(r"globaltimer_ns\(\)\s*-\s*t0\s*>\s*\w", body), body[:80]
        assert "return false" in body, body[:80]
    assert "*c.abort" in allowed[0] and "raise_abort" in allowed[0]
    definition = _function_body(sm, "mbar_try_wait")
    for name, src in srcs.items():
        rest = src
        if name == "sm100.cuh":
            for body in allowed + [definition]:
                rest = rest.replace(body, "")
        calls = re.findall(r"\bmbar_try_wait\s*\(", rest)
        assert not calls, f"{name}: mbar_try_wait polled outside the bounded waits"


def test_no_trap_or_device_assert():
    for name, src in _sources().items():
        assert "__trap" not in src and not re.search(r"\btrap\s*;", src), name
        assert not re.search(r"(?<!static_)\bassert\s*\(", src), name
