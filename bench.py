"""Benchmark of the exact-attention hot path on B200.

One step = one pass over the whole path, one launch per workload, each timed with CUDA
events after its own L2 flush:
  * fa_fwd on tiny (B=1 H=2 N=128 d=64 fp16, non-causal), mha2k (B=8 H=12 N=2048 d=64
    fp16, causal), gqa8k (B=1 Hq=32 Hkv=8 N=8192 d=128 bf16, causal) and gqa32k (the same
    at N=32768), each writing O and LSE;
  * fa_decode on the GQA decode workload B=64 Hq=32 Hkv=8 d=128 bf16, kv_len ~ U[512,4096].
`value` is the long-context GQA prefill's throughput in TFLOP/s (algorithmic,
causal-adjusted FLOPs: 4*d per visible query-key pair); every workload's throughput,
spread and roofline is in `configs` (TFLOP/s for the prefills, KV-read GB/s for the decode).

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun (N > 1) each rank runs an independent replica (the path needs no
collective); the barrier and the max-over-ranks time are the only communication.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import (WORKLOADS, decode_kv_bytes, fwd_flops, make_decode_inputs,  # noqa: E402
                       make_fp8_inputs, make_fwd_inputs, make_page_table, paginate)

METRIC = "attn fwd TFLOP/s & % BF16 TC peak; decode KV-read GB/s & % HBM peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
L2_NOTE = ("flushed before each step: a 256 MiB write, then a 256 MiB read so that the lines "
           "left in L2 are clean; decode caches exceed L2")
# ex2.approx.f32 results per clock per SM, measured on this machine's B200s with a throughput
# probe (independent chains, 4-32 warps per SM); f16x2/bf16x2 forms give the same rate.
MUFU_EX2_PER_CLK_SM = 16.0
# One step runs every workload once, in this order, then the decode; the headline value is
# the long-context GQA prefill.
FWD_ORDER = ["tiny", "mha2k", "gqa8k", "gqa32k"]
HEADLINE = "gqa32k"


def max_over_ranks(local_ms, world: int, device):
    """Per-rank device times (a list of floats) reduced to their maximum over all ranks.
    Every rank calls this at the same point with the same list length; with one rank it
    returns the list unchanged. The job is as slow as its slowest rank."""
    import torch
    t = torch.tensor([float(x) for x in local_ms], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def spread_ms(ms):
    """Mean, median, 10th and 90th percentile and extremes of per-launch times (ms)."""
    xs = sorted(float(x) for x in ms)
    n = len(xs)

    def pct(p):
        if n == 1:
            return xs[0]
        pos = p * (n - 1)
        lo = int(math.floor(pos))
        hi = min(lo + 1, n - 1)
        return xs[lo] + (xs[hi] - xs[lo]) * (pos - lo)

    return {"mean": sum(xs) / n, "median": pct(0.5), "p10": pct(0.1), "p90": pct(0.9),
            "min": xs[0], "max": xs[-1], "n": n}


def job_rate(world: int, steps: int, work_per_step: float, max_ms: float) -> float:
    """Whole-job throughput: every rank did `steps` steps of `work_per_step` units (weak
    scaling, replicas), and the job took the slowest rank's `max_ms`."""
    return world * steps * work_per_step / (max_ms * 1e-3)


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu capture for (kernel, workload), or None
    if there is none or the kernel sources changed since it was taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            cap = json.load(f)["captures"][f"{kernel}|{workload}"]
        h = hashlib.sha256()
        for src in cap["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        if h.hexdigest()[:16] != cap["sources_sha256_16"]:
            return None
        return cap["dram_read_bytes"] + cap["dram_write_bytes"]
    except Exception:
        return None


def make_l2_flush(dev):
    """A callable that empties L2 (126 MB) of everything a timed launch could reuse.

    It writes a 256 MiB buffer and then reads another one. The read matters: after the
    write alone, L2 is full of dirty lines, and whichever timed kernel runs next pays for
    writing them back (about 19 us of HBM time for a bandwidth-bound kernel). After the
    read, the lines in L2 are clean and unrelated to the workload."""
    import torch
    wbuf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    # float32, so that the sum reduces it in place (an integer sum would first widen the
    # whole buffer to int64, a 512 MiB write that leaves dirty lines behind).
    rbuf = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush():
        wbuf.zero_()
        rbuf.sum()

    return flush


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------------------
# Clock sampling during the timed region (NVML, read-only)
# ---------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = [("gpu_idle", 0x1), ("applications_clocks_setting", 0x2), ("sw_power_cap", 0x4),
               ("hw_slowdown", 0x8), ("sync_boost", 0x10), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80)]

    def __init__(self, cuda_index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.error = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = self._handle(cuda_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report the clocks as unavailable
            self.nvml, self.error = None, f"{type(e).__name__}: {e}"

    def _handle(self, idx):
        import torch
        pynvml = self.nvml
        try:
            uuid = str(torch.cuda.get_device_properties(idx).uuid)
            for u in (uuid, "GPU-" + uuid):
                try:
                    return pynvml.nvmlDeviceGetHandleByUUID(u)
                except Exception:
                    pass
        except Exception:
            pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            try:
                idx = int(vis.split(",")[idx])
            except Exception:
                pass
        return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        p = self.nvml
        get_reasons = getattr(p, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(p, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                self.samples.append(p.nvmlDeviceGetClockInfo(self.handle, p.NVML_CLOCK_SM))
                self.reasons |= int(get_reasons(self.handle))
            except Exception as e:
                self.error = str(e)
            time.sleep(self.period)

    def start(self):
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "note": self.error or "no samples"}
        names = [n for n, bit in self.REASONS if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------
# CPU oracle timings (the float64 oracle as it stands, on this host's cores)
# ---------------------------------------------------------------------------------------
def host_cpu():
    """Host CPU model name (lscpu) and the cores this process may run on."""
    model = None
    try:
        import subprocess
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.lower().startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except Exception:
        pass
    return {"model_name": model, "cores": len(os.sched_getaffinity(0))}


def causal_pairs(rows, Nq: int, Nk: int) -> int:
    """Visible (query, key) pairs of the given query rows under the bottom-right causal mask."""
    off = Nk - Nq
    return int(sum(max(0, min(Nk, int(i) + off + 1)) for i in rows))


def oracle_rows_time(w, rows, heads, q=None, k=None, v=None):
    """Time the oracle on `rows` of each (batch, head) in `heads`; returns (seconds,
    algorithmic FLOPs of that work)."""
    import numpy as np
    from oracle import attention_rows_f64
    if q is None:
        q, k, v = make_fwd_inputs(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, w.seed)
    rows = np.asarray(rows, dtype=np.int64)
    pairs = causal_pairs(rows, w.N, w.N) if w.causal else len(rows) * w.N
    t0 = time.perf_counter()
    for b, h in heads:
        attention_rows_f64(q, k, v, w.causal, w.scale, b, h, rows)
    return time.perf_counter() - t0, 4.0 * w.d * pairs * len(heads)


def oracle_baselines(budget_s: float):
    """Per-workload CPU oracle figures on bounded samples (about 10 s of host time in all):
    tiny in full; mha2k on as many whole (batch, head) problems as a quarter of `budget_s`
    allows; gqa8k on 1024 rows of one head; gqa32k on 256 seeded rows of one head (rows 0,
    1, 127, 128 and N-1 among them); the decode on 16 of its 64 sequences. Full-size times
    are extrapolated from the samples and labelled estimates."""
    import numpy as np
    from oracle import decode_f64
    host = host_cpu()
    res = {}
    w = WORKLOADS["tiny"]
    el, fl = oracle_rows_time(w, np.arange(w.N), [(b, h) for b in range(w.B) for h in range(w.Hq)])
    res["tiny"] = {"value": fl / el / 1e12, "unit": "TFLOP/s", "seconds": el,
                   "sample": "the whole workload"}
    w = WORKLOADS["mha2k"]
    q, k, v = make_fwd_inputs(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, w.seed)
    heads, el, fl = 0, 0.0, 0.0
    order = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    while heads < len(order) and el < 0.25 * budget_s:
        e, f = oracle_rows_time(w, np.arange(w.N), [order[heads]], q, k, v)
        el, fl, heads = el + e, fl + f, heads + 1
    res["mha2k"] = {"value": fl / el / 1e12, "unit": "TFLOP/s", "seconds": el,
                    "sample": f"{heads} of {len(order)} whole (batch, head) problems",
                    "full_workload_seconds_estimate": el * len(order) / heads}
    w = WORKLOADS["gqa8k"]
    rows = np.concatenate([np.arange(r, r + 256) for r in (0, w.N // 4, w.N // 2, w.N - 256)])
    el, fl = oracle_rows_time(w, rows, [(0, 0)])
    res["gqa8k"] = {"value": fl / el / 1e12, "unit": "TFLOP/s", "seconds": el,
                    "sample": f"{len(rows)} rows of one head (four 256-row blocks spread over the "
                              f"sequence) of {w.Hq} heads",
                    "full_workload_seconds_estimate": el / len(rows) * w.N * w.Hq,
                    "estimate_note": "estimate: the sample's time per row times all rows of all heads"}
    w = WORKLOADS["gqa32k"]
    rows = np.unique(np.concatenate([[0, 1, 127, 128, w.N - 1],
                                     np.random.default_rng(w.N).choice(w.N, 251, replace=False)]))
    el, fl = oracle_rows_time(w, rows, [(0, 0)])
    per_row = el / len(rows)
    res["gqa32k"] = {"value": fl / el / 1e12, "unit": "TFLOP/s", "seconds": el,
                     "sample": f"{len(rows)} seeded rows (0, 1, 127, 128, N-1 among them) of one head",
                     "full_workload_seconds_estimate": per_row * w.N * w.Hq,
                     "estimate_note": "estimate: the sample's time per row times all rows of all "
                                      "heads (the oracle forms every row over all N keys)"}
    w = WORKLOADS["decode"]
    kv_lens, dq, kc, vc = make_decode_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.dtype, w.kv_len_lo,
                                             w.kv_len_hi, w.seed)
    nb = 16
    t0 = time.perf_counter()
    decode_f64(dq[:nb], kc[:nb], vc[:nb], kv_lens[:nb], w.scale)
    el = time.perf_counter() - t0
    res["decode"] = {"value": decode_kv_bytes(kv_lens[:nb], w.Hkv, w.d) / el / 1e9, "unit": "GB/s",
                     "seconds": el, "sample": f"the first {nb} of {w.B} sequences",
                     "full_workload_seconds_estimate": el * decode_kv_bytes(kv_lens, w.Hkv, w.d)
                     / decode_kv_bytes(kv_lens[:nb], w.Hkv, w.d),
                     "estimate_note": "estimate: scaled by the KV bytes of all sequences"}
    for r in res.values():
        r.update({"kind": "oracle", "cores": host["cores"]})
    return res, host


def run_reference(args):
    """Reference arm: the float64 CPU oracle as it stands, on rank 0 only, on the headline
    workload (long-context GQA prefill): each step is 256 seeded query rows of one head
    (rows 0, 1, 127, 128 and N-1 among them), heads taken in turn."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    w = WORKLOADS[HEADLINE]
    q, k, v = make_fwd_inputs(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, w.seed)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, w.N - 1],
                                     np.random.default_rng(w.N).choice(w.N, 251, replace=False)]))

    def step(i):
        return oracle_rows_time(w, rows, [(0, i % w.Hq)], q, k, v)

    for i in range(args.warmup):
        step(i)
    el, fl = 0.0, 0.0
    for i in range(args.steps):
        e, f = step(args.warmup + i)
        el, fl = el + e, fl + f
    val = fl / el / 1e12
    host = host_cpu()
    sample = f"{len(rows)} seeded query rows of one head per step, heads in turn"
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.describe(), "parallelism": "single process, host cores",
                       "sample_per_step": sample},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": host["cores"], "kind": "oracle",
                             "sample": sample, "host_cpu": host["model_name"]},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------
def run_ours(args):
    import torch
    import torch.distributed as dist
    import io_aware_exact_28_b200 as fa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    peaks, peak_src = load_peaks()
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    l2_flush = make_l2_flush(dev)

    # Inputs (seeded, CPU-generated), resident on the device before timing. One entry per
    # workload: the call, its work per launch and what bounds it.
    calls = []
    for name in FWD_ORDER:
        w = WORKLOADS[name]
        q, k, v = (t.to(dev) for t in make_fwd_inputs(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, w.seed))
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)

        def call(q=q, k=k, v=v, o=o, lse=lse, w=w):
            fa.fwd(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse)

        calls.append({"name": name, "w": w, "call": call, "kind": "fwd",
                      "work": fwd_flops(w.B, w.Hq, w.N, w.N, w.d, w.causal),
                      "bytes": 2 * (2 * q.numel() + 2 * k.numel()) + 4 * lse.numel(),
                      "tensors": (q, k, v, o, lse)})
    wd = WORKLOADS["decode"]
    kv_lens_cpu, dq, kc, vc = make_decode_inputs(wd.B, wd.Hq, wd.Hkv, wd.N, wd.d, wd.dtype,
                                                 wd.kv_len_lo, wd.kv_len_hi, wd.seed)
    kv_lens, dq, kc, vc = kv_lens_cpu.to(dev), dq.to(dev), kc.to(dev), vc.to(dev)
    do = torch.empty_like(dq)
    dlse = torch.empty((wd.B, wd.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.decode_workspace_bytes(wd.B, wd.Hq, wd.N, wd.d), dtype=torch.uint8, device=dev)

    def dec_call():
        fa.decode(dq, kc, vc, kv_lens, scale=wd.scale, out=do, lse=dlse, workspace=ws)

    kv_bytes = decode_kv_bytes(kv_lens_cpu, wd.Hkv, wd.d)
    calls.append({"name": "decode", "w": wd, "call": dec_call, "kind": "decode",
                  "work": kv_bytes + 2 * (dq.numel() + do.numel()) + 4 * dlse.numel(),
                  "kv_bytes": kv_bytes})
    dec_kernel = "fa_decode_tc_kernel" if wd.d == 128 else "fa_decode_split_kernel"

    def step(ev=None):
        for i, c in enumerate(calls):
            l2_flush()                # every kernel starts from a cold, clean L2
            if ev is not None:
                ev[i][0].record()
            c["call"]()
            if ev is not None:
                ev[i][1].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fa.device_status() != fa.FA_OK:
        raise RuntimeError("device status not OK after warm-up")

    K = args.steps
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in calls] for _ in range(K)]
    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    for s_ in range(K):
        step(evs[s_])
    torch.cuda.synchronize()
    sampler.stop()
    if world > 1:
        dist.barrier()
    # per-launch times, then the max over ranks of every number (same list length everywhere)
    per = [[evs[s_][i][0].elapsed_time(evs[s_][i][1]) for s_ in range(K)] for i in range(len(calls))]
    flat = max_over_ranks([x for row in per for x in row], world, dev)
    per = [flat[i * K:(i + 1) * K] for i in range(len(calls))]
    status = fa.device_status()
    clocks = sampler.summary()
    sm_mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz")

    configs = []
    for c, ms in zip(calls, per):
        w, tot = c["w"], sum(ms)
        sp = spread_ms(ms)
        rate = job_rate(world, K, c["work"], tot)          # per second, whole job
        per_launch_rate = c["work"] / (sp["mean"] * 1e-3)
        entry = {"name": c["name"], "workload": w.describe(), "ms_per_launch": sp, "launches": K}
        if c["kind"] == "fwd":
            entry.update({"value": rate / 1e12, "unit": "TFLOP/s",
                          "value_at_median": c["work"] / (sp["median"] * 1e-3) / 1e12 * world,
                          "algorithmic_flops_per_launch": c["work"],
                          "algorithmic_bytes_per_launch": c["bytes"]})
            roof = {"kernel": "fa_fwd_kernel", "bound": "tensor", "achieved": per_launch_rate / 1e12,
                    "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": per_launch_rate / 1e12 / peaks["bf16_tflops"],
                    "frac_of_sustained": per_launch_rate / 1e12 / peaks["bf16_tflops_sustained"],
                    "frac_of_spec_2250": per_launch_rate / 1e12 / 2250.0,
                    "traffic": measured_traffic("fa_fwd_kernel", c["name"]),
                    "peak_source": f"{peak_src} dense bf16 burst (fp16 has the same dense rate)"}
            if sm_mhz:
                exps = c["work"] / (4.0 * w.d)
                peak_exps = MUFU_EX2_PER_CLK_SM * n_sm * sm_mhz * 1e6
                roof["exp_unit"] = {"bound": "alu", "unit": "exp2/s",
                                    "achieved": exps / (sp["mean"] * 1e-3), "peak": peak_exps,
                                    "frac": exps / (sp["mean"] * 1e-3) / peak_exps,
                                    "peak_source": f"measured {MUFU_EX2_PER_CLK_SM} ex2.approx/clk/SM x "
                                                   f"{n_sm} SMs x sampled {sm_mhz} MHz"}
            if c["name"] == "tiny":
                roof["note"] = "launch-latency bound: report the microseconds, not the fraction"
        else:
            entry.update({"value": rate / 1e9, "unit": "GB/s",
                          "value_at_median": c["work"] / (sp["median"] * 1e-3) / 1e9 * world,
                          "algorithmic_bytes_per_launch": c["work"], "kv_bytes_per_launch": c["kv_bytes"]})
            roof = {"kernel": f"fa_decode ({dec_kernel} + fa_decode_combine_kernel)", "bound": "hbm",
                    "achieved": per_launch_rate / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": per_launch_rate / 1e9 / peaks["hbm_gbs"],
                    "frac_of_spec_8000": per_launch_rate / 1e9 / 8000.0,
                    "traffic": measured_traffic(dec_kernel, "decode"),
                    "traffic_note": f"{dec_kernel} only (the combine kernel moves ~2% more)",
                    "peak_source": f"{peak_src} HBM copy bandwidth"}
        entry["roofline"] = roof
        configs.append(entry)
    head = next(e for e in configs if e["name"] == HEADLINE)
    dominant = max(configs, key=lambda e: e["ms_per_launch"]["mean"])["roofline"]

    # End to end through the public API for the headline workload: host (pinned) inputs in,
    # host outputs back, every step. Copies run on their own streams with double-buffered
    # device tensors, so the upload of step i+1 and the download of step i overlap the
    # forward of step i (as a serving loop would); the copy bytes per step are unchanged.
    e2e = None
    if not args.no_e2e:
        hc = next(c for c in calls if c["name"] == HEADLINE)
        w = hc["w"]
        q, k, v, o, lse = hc["tensors"]
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
        ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
        hl = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(2)]
        dq2 = [torch.empty_like(q) for _ in range(2)]
        dk2 = [torch.empty_like(k) for _ in range(2)]
        dv2 = [torch.empty_like(v) for _ in range(2)]
        do2 = [torch.empty_like(o) for _ in range(2)]
        dl2 = [torch.empty_like(lse) for _ in range(2)]
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        e_in = [torch.cuda.Event() for _ in range(2)]
        e_cmp = [torch.cuda.Event() for _ in range(2)]
        e_out = [torch.cuda.Event() for _ in range(2)]
        E = max(3, min(K, args.e2e_steps))

        def e2e_step(n):
            bi = n & 1
            with torch.cuda.stream(s_in):
                if n >= 2:
                    s_in.wait_event(e_cmp[bi])      # step n-2 has read these inputs
                dq2[bi].copy_(hq, non_blocking=True)
                dk2[bi].copy_(hk, non_blocking=True)
                dv2[bi].copy_(hv, non_blocking=True)
                e_in[bi].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(e_in[bi])
                if n >= 2:
                    s_cmp.wait_event(e_out[bi])     # step n-2's outputs are on the host
                fa.fwd(dq2[bi], dk2[bi], dv2[bi], causal=w.causal, scale=w.scale, out=do2[bi],
                       lse=dl2[bi], stream=s_cmp)
                e_cmp[bi].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(e_cmp[bi])
                ho[bi].copy_(do2[bi], non_blocking=True)
                hl[bi].copy_(dl2[bi], non_blocking=True)
                e_out[bi].record(s_out)

        for n in range(4):
            e2e_step(n)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(s_in)
        for n in range(E):
            e2e_step(n)
        s_in.wait_stream(s_out)
        s_in.wait_stream(s_cmp)
        s1.record(s_in)
        torch.cuda.synchronize()
        (e2e_ms,) = max_over_ranks([s0.elapsed_time(s1)], world, dev)
        e2e = {"value": job_rate(world, E, hc["work"], e2e_ms) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": 2 * (q.numel() + k.numel() + v.numel()),
               "d2h_bytes_per_step": 2 * o.numel() + 4 * lse.numel(), "steps": E,
               "workload": w.describe(),
               "path": "fa.fwd (C ABI fa_fwd) with pinned host buffers; copies on separate "
                       "streams, double-buffered, overlapping the previous/next step"}

    cpu, host = None, None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        per_cfg, host = oracle_baselines(args.cpu_budget_s)
        for e in configs:
            e["cpu_baseline"] = per_cfg[e["name"]]
        cpu = dict(per_cfg[HEADLINE])
        cpu["host_cpu"] = host["model_name"]

    if rank == 0:
        ms_step = sum(sum(ms) for ms in per) / K
        line = {
            "metric": METRIC, "value": head["value"], "unit": "TFLOP/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": head_dtype(), "data": "synthetic",
            "config": {"workload": WORKLOADS[HEADLINE].describe(),
                       "step": "one launch of each workload: " + ", ".join(
                           WORKLOADS[n].describe() for n in FWD_ORDER + ["decode"]),
                       "l2": L2_NOTE,
                       "parallelism": "replicas" if world > 1 else "single GPU",
                       "value_is": "long-context GQA causal prefill TFLOP/s (causal-adjusted "
                                   "algorithmic FLOPs); every workload's figure is in configs"},
            "configs": configs,
            "roofline": dominant, "rooflines": [e["roofline"] for e in configs],
            "e2e": e2e, "cpu_baseline": cpu, "host_cpu": host,
            "gpu_launches": K * (len(FWD_ORDER) + (3 if dec_kernel == "fa_decode_tc_kernel" else 2)),
            "gpu_launches_note": (f"per step: fa_fwd_kernel x {len(FWD_ORDER)} + "
                                  + ("fa_decode_ticket_reset_kernel + " if dec_kernel == "fa_decode_tc_kernel" else "")
                                  + f"{dec_kernel} + fa_decode_combine_kernel"),
            "clocks": clocks,
            "device_status": fa.status_string(status),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def head_dtype():
    return WORKLOADS[HEADLINE].dtype


def run_single_kernel(args):
    """--only fwd|decode: allocate and launch one entry point alone (warm-up, then K timed
    launches). Used for profiler captures, where a small device footprint matters."""
    import torch
    import io_aware_exact_28_b200 as fa
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    if args.only == "fwd":
        w = WORKLOADS[args.workload]
        q, k, v = (t.to(dev) for t in make_fwd_inputs(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, w.seed))
        o, lse = torch.empty_like(q), torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
        work = fwd_flops(w.B, w.Hq, w.N, w.N, w.d, w.causal) / 1e12
        unit = "TFLOP/s"

        def call():
            fa.fwd(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse)
    elif args.only == "bwd":
        # Backward pass (fa_bwd) of the workload, with fa_fwd's O and LSE as its inputs.
        # Algorithmic FLOPs: 2.5x the forward's (five N^2 d products instead of two).
        w = WORKLOADS[args.workload]
        q, k, v = (t.to(dev) for t in make_fwd_inputs(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, w.seed))
        gen = torch.Generator(device=dev).manual_seed(w.seed + 1)
        dout = torch.randn(q.shape, generator=gen, device=dev, dtype=torch.float32).to(q.dtype)
        o, lse = fa.fwd(q, k, v, causal=w.causal, scale=w.scale)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(fa.bwd_workspace_bytes(w.B, w.Hq, w.N), dtype=torch.uint8, device=dev)
        work = 2.5 * fwd_flops(w.B, w.Hq, w.N, w.N, w.d, w.causal) / 1e12
        unit = "TFLOP/s"

        def call():
            fa.bwd(q, k, v, o, lse, dout, causal=w.causal, scale=w.scale, dq=dq, dk=dk, dv=dv,
                   workspace=ws)
    elif args.only == "chunked":
        # Chunked prefill: the workload's sequence in --chunk-token pieces, each attending
        # to the cache prefix up to its own end (fa_fwd_kvcache); same causal FLOPs.
        w = WORKLOADS[args.workload]
        q, k, v = (t.to(dev) for t in make_fwd_inputs(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, w.seed))
        o, lse = torch.empty_like(q), torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
        work = fwd_flops(w.B, w.Hq, w.N, w.N, w.d, True) / 1e12
        unit = "TFLOP/s"
        C = args.chunk
        qs = [q[:, :, i:i + C].contiguous() for i in range(0, w.N, C)]
        outs = [torch.empty_like(x) for x in qs]

        def call():
            for n, i in enumerate(range(0, w.N, C)):
                fa.fwd_kvcache(qs[n], k, v, min(i + C, w.N), causal=True, scale=w.scale, out=outs[n],
                               return_lse=False)
    elif args.only == "fwd_fp8":
        # The workload's shape with E4M3 Q, K, V (fa_fwd_fp8, bf16 output); same causal FLOPs.
        w = WORKLOADS[args.workload]
        q8, k8, v8, dq_, dk_, dv_ = make_fp8_inputs(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.seed)
        q8, k8, v8 = q8.to(dev), k8.to(dev), v8.to(dev)
        o = torch.empty(q8.shape, dtype=torch.bfloat16, device=dev)
        lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
        work = fwd_flops(w.B, w.Hq, w.N, w.N, w.d, w.causal) / 1e12
        unit = "TFLOP/s"

        def call():
            fa.fwd_fp8(q8, k8, v8, dq_, dk_, dv_, causal=w.causal, scale=w.scale, out=o, lse=lse)
    elif args.only == "fwd_varlen":
        # A ragged batch with the workload's head shape: sequences of different lengths
        # (--varlen-lens, each a full causal prefill) in one fa_fwd_kvcache call with
        # per-sequence lengths; FLOPs are the sum of each sequence's causal FLOPs.
        w = WORKLOADS[args.workload]
        lens = [int(x) for x in args.varlen_lens.split(",")]
        B, cap = len(lens), max(lens)
        q, k, v = (t.to(dev) for t in make_fwd_inputs(B, w.Hq, w.Hkv, cap, cap, w.d, w.dtype, w.seed))
        o, lse = torch.empty_like(q), torch.empty((B, w.Hq, cap), dtype=torch.float32, device=dev)
        ln = torch.tensor(lens, dtype=torch.int32, device=dev)
        work = sum(fwd_flops(1, w.Hq, n, n, w.d, True) for n in lens) / 1e12
        unit = "TFLOP/s"

        def call():
            fa.fwd_kvcache(q, k, v, cap, causal=True, scale=w.scale, out=o, lse=lse, q_lens=ln,
                           kv_lens=ln)
    elif args.only == "fwd_paged":
        # Prefill of the workload with K and V in a page pool (fa_fwd_paged), pages drawn by
        # a seeded random table; same causal FLOPs as --only fwd.
        w = WORKLOADS[args.workload]
        q, k, v = make_fwd_inputs(w.B, w.Hq, w.Hkv, w.N, w.N, w.d, w.dtype, w.seed)
        ps = args.page_size
        lens = torch.full((w.B,), w.N)
        table, n_pages = make_page_table(lens, ps, (w.N + ps - 1) // ps, seed=w.seed)
        kp, vp = paginate(k, table, lens, ps, n_pages), paginate(v, table, lens, ps, n_pages)
        q, kp, vp, table = q.to(dev), kp.to(dev), vp.to(dev), table.to(dev)
        o, lse = torch.empty_like(q), torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
        work = fwd_flops(w.B, w.Hq, w.N, w.N, w.d, w.causal) / 1e12
        unit = "TFLOP/s"

        def call():
            fa.fwd_paged(q, kp, vp, table, w.N, causal=w.causal, scale=w.scale, out=o, lse=lse)
    elif args.only == "decode_paged":
        # The decode workload with its cache in a page pool (fa_decode_paged).
        w = WORKLOADS[args.decode_workload]
        kv_cpu, dq, kc, vc = make_decode_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.dtype, w.kv_len_lo,
                                                w.kv_len_hi, w.seed)
        ps = args.page_size
        table, n_pages = make_page_table(kv_cpu, ps, w.N // ps, seed=w.seed)
        kp, vp = paginate(kc, table, kv_cpu, ps, n_pages), paginate(vc, table, kv_cpu, ps, n_pages)
        del kc, vc
        kv_lens, dq, kp, vp, table = kv_cpu.to(dev), dq.to(dev), kp.to(dev), vp.to(dev), table.to(dev)
        do, dlse = torch.empty_like(dq), torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
        ws = torch.empty(fa.decode_workspace_bytes(w.B, w.Hq, w.N, w.d), dtype=torch.uint8, device=dev)
        work = (decode_kv_bytes(kv_cpu, w.Hkv, w.d) + 4 * dq.numel() + 4 * dlse.numel()) / 1e9
        unit = "GB/s"

        def call():
            fa.decode_paged(dq, kp, vp, table, kv_lens, scale=w.scale, out=do, lse=dlse, workspace=ws)
    else:
        w = WORKLOADS[args.decode_workload]
        kv_cpu, dq, kc, vc = make_decode_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.dtype, w.kv_len_lo,
                                                w.kv_len_hi, w.seed)
        kv_lens, dq, kc, vc = kv_cpu.to(dev), dq.to(dev), kc.to(dev), vc.to(dev)
        do, dlse = torch.empty_like(dq), torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
        ws = torch.empty(fa.decode_workspace_bytes(w.B, w.Hq, w.N, w.d), dtype=torch.uint8, device=dev)
        work = (decode_kv_bytes(kv_cpu, w.Hkv, w.d) + 4 * dq.numel() + 4 * dlse.numel()) / 1e9
        unit = "GB/s"

        def call():
            fa.decode(dq, kc, vc, kv_lens, scale=w.scale, out=do, lse=dlse, workspace=ws)
    l2_flush = make_l2_flush(dev)
    for _ in range(args.warmup):
        l2_flush()
        call()
    torch.cuda.synchronize()
    ms = []
    for _ in range(args.steps):
        l2_flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    status = fa.status_string(fa.device_status())
    avg = sum(ms) / len(ms)
    spread = spread_ms(ms)
    print(json.dumps({"only": args.only, "workload": w.describe(),
                      **({"chunk": args.chunk} if args.only == "chunked" else {}),
                      **({"page_size": args.page_size} if "paged" in args.only else {}),
                      **({"lens": args.varlen_lens} if args.only == "fwd_varlen" else {}), "ms_per_launch": avg,
                      "value": work / (avg * 1e-3), "value_at_median": work / (spread["median"] * 1e-3),
                      "unit": unit, "ms_spread": spread, "device_status": status}))
    return 0 if status == "FA_OK" else 1


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--only", choices=["fwd", "decode", "chunked", "bwd", "fwd_paged", "decode_paged",
                                       "fwd_fp8", "fwd_varlen"],
                    default=None,
                    help="launch one entry point alone (profiling helper; prints its own line)")
    ap.add_argument("--gpus", type=int, default=1,
                    help="ranks of the job (one per GPU, launched by torchrun when > 1)")
    ap.add_argument("--steps", type=int, default=50, help="timed steps")
    ap.add_argument("--warmup", type=int, default=10, help="untimed warm-up steps (at least 3)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours",
                    help="reference: time the float64 CPU oracle on the headline workload")
    ap.add_argument("--workload", default="mha2k", choices=[k for k, v in WORKLOADS.items() if v.kind == "fwd"],
                    help="--only: the prefill workload")
    ap.add_argument("--chunk", type=int, default=1024, help="--only chunked: tokens per chunk")
    ap.add_argument("--page-size", type=int, default=64, help="--only *_paged: tokens per page")
    ap.add_argument("--varlen-lens", default="8192,6144,3072,1024",
                    help="--only fwd_varlen: comma-separated sequence lengths of the batch")
    ap.add_argument("--decode-workload", default="decode", help="--only decode*: the decode workload")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end run from pinned host buffers")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the CPU oracle timing")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0,
                    help="host seconds the CPU oracle timing may take in all")
    ap.add_argument("--e2e-steps", type=int, default=20, help="steps of the end-to-end run")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)   # at least 3 untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    if args.only:
        return run_single_kernel(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
