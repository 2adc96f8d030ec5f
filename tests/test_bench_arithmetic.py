"""The measurement arithmetic behind the reported numbers, checked on the CPU against
counting by brute force:

* algorithmic FLOPs of a forward call are 4 d per visible (query, key) pair (QK^T and
  P.V, two FLOPs per multiply-add), with the bottom-right causal rule;
* the visible pairs of a subset of query rows (the CPU oracle samples);
* the K and V bytes a decode step must read;
* the per-launch timing spread (linear-interpolated percentiles);
* the DRAM traffic taken from the committed ncu captures, which counts only while the
  hash of the kernel sources it was taken on still matches;
* the clock record (median SM clock, named throttle reasons) read from NVML, here a
  read-only stand-in.
"""
import hashlib
import json
import math
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import WORKLOADS, decode_kv_bytes, fwd_flops  # noqa: E402


def visible_pairs_brute(rows, Nq, Nk, causal):
    n = 0
    for i in rows:
        for j in range(Nk):
            if not causal or j - i <= Nk - Nq:
                n += 1
    return n


@pytest.mark.parametrize("Nq,Nk", [(1, 1), (5, 5), (3, 8), (8, 3), (17, 40), (40, 17), (64, 64)])
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_flops_count_visible_pairs(Nq, Nk, causal):
    B, Hq, d = 2, 3, 8
    pairs = visible_pairs_brute(range(Nq), Nq, Nk, causal)
    assert fwd_flops(B, Hq, Nq, Nk, d, causal) == 4.0 * d * pairs * B * Hq


def test_fwd_flops_closed_forms_of_the_workloads():
    """Square causal problems have N (N + 1) / 2 visible pairs per head."""
    for w in WORKLOADS.values():
        if w.kind == "decode":
            continue
        pairs = w.N * (w.N + 1) // 2 if w.causal else w.N * w.N
        assert fwd_flops(w.B, w.Hq, w.N, w.N, w.d, w.causal) == 4.0 * w.d * pairs * w.B * w.Hq
    mha = WORKLOADS["mha2k"]
    assert fwd_flops(mha.B, mha.Hq, mha.N, mha.N, mha.d, True) == 51_564_773_376.0


@pytest.mark.parametrize("Nq,Nk", [(7, 7), (4, 9), (9, 4)])
def test_causal_pairs_of_sampled_rows(Nq, Nk):
    rng = np.random.default_rng(Nq * 31 + Nk)
    for _ in range(5):
        rows = rng.choice(Nq, size=rng.integers(1, Nq + 1), replace=False)
        assert bench.causal_pairs(rows, Nq, Nk) == visible_pairs_brute(rows, Nq, Nk, True)
    assert bench.causal_pairs(range(Nq), Nq, Nk) * 4 * 8 == fwd_flops(1, 1, Nq, Nk, 8, True)


def test_decode_kv_bytes():
    lens = torch.tensor([0, 1, 517, 4096], dtype=torch.int32)
    Hkv, d = 8, 128
    brute = 0
    for n in lens.tolist():
        brute += n * Hkv * d * 2 * 2            # K and V rows, 16-bit elements
    assert decode_kv_bytes(lens, Hkv, d) == brute
    assert decode_kv_bytes(lens, Hkv, d, elem_bytes=1) == brute // 2


def test_spread_matches_linear_percentiles():
    rng = np.random.default_rng(3)
    for n in (1, 2, 7, 50):
        ms = rng.uniform(0.1, 2.0, n)
        s = bench.spread_ms(ms)
        assert s["n"] == n and s["min"] == ms.min() and s["max"] == ms.max()
        assert s["mean"] == pytest.approx(ms.mean(), rel=1e-12)
        for key, p in (("median", 50), ("p10", 10), ("p90", 90)):
            assert s[key] == pytest.approx(np.percentile(ms, p), rel=1e-12), (n, key)


def test_measured_traffic_follows_the_source_hash():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        caps = json.load(f)["captures"]
    assert caps
    assert bench.measured_traffic("no_such_kernel", "mha2k") is None
    for key, cap in caps.items():
        kernel, workload = key.split("|")
        h = hashlib.sha256()
        for src in cap["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        want = cap["dram_read_bytes"] + cap["dram_write_bytes"] \
            if h.hexdigest()[:16] == cap["sources_sha256_16"] else None
        assert bench.measured_traffic(kernel, workload) == want, key


def test_job_rate_is_whole_job_work_over_the_slowest_rank():
    assert bench.job_rate(4, 20, 1.5, 10.0) == pytest.approx(4 * 20 * 1.5 / 0.010)
    assert math.isclose(bench.job_rate(1, 1, 1.0, 1000.0), 1.0)


class _FakeNvml:
    """Read-only NVML stand-in: a fixed clock sequence and throttle-reason bitmask."""
    NVML_CLOCK_SM = 1

    def __init__(self, clocks, reasons):
        self.clocks, self.reasons, self.i = list(clocks), reasons, 0

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByUUID(self, u):
        raise RuntimeError("no uuid")

    def nvmlDeviceGetHandleByIndex(self, idx):
        return ("handle", idx)

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        c = self.clocks[min(self.i, len(self.clocks) - 1)]
        self.i += 1
        return c

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.reasons


def test_clock_sampler_reports_median_and_named_reasons(monkeypatch):
    fake = _FakeNvml([1700, 1755, 1740, 1965, 1725], 0x1 | 0x4 | 0x8)
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    cs = bench.ClockSampler(0, period_s=0.001)
    assert cs.nvml is fake and cs.max_mhz == 1965
    cs.start()
    import time
    t0 = time.monotonic()
    while len(cs.samples) < 5 and time.monotonic() - t0 < 2.0:
        time.sleep(0.005)
    cs.stop()
    s = cs.summary()
    assert s["samples"] >= 5 and s["sm_max_mhz"] == 1965
    assert s["sm_mhz"] == float(np.median([fake.clocks[min(i, 4)] for i in range(s["samples"])]))
    assert s["reasons"] == ["sw_power_cap", "hw_slowdown"]      # gpu_idle is not reported


def test_clock_sampler_without_nvml_reports_no_samples(monkeypatch):
    class Broken:
        def nvmlInit(self):
            raise RuntimeError("NVML not found")
    monkeypatch.setitem(sys.modules, "pynvml", Broken())
    cs = bench.ClockSampler(0)
    cs.start()
    cs.stop()
    s = cs.summary()
    assert s["samples"] == 0 and s["sm_mhz"] is None and "NVML not found" in s["note"]
