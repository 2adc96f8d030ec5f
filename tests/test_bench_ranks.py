"""World-size-2 CPU checks (gloo) of the multi-rank bench logic. The path does not shard
(replicas only): ranks run independent copies of the step, and the only collectives are a
barrier and the max over ranks of the device times. These tests run that logic on two CPU
processes: every rank gets the slowest rank's time, whole-job throughput counts every
rank's work against it, and the reference arm runs on rank 0 only."""
import json
import os
import socket
import subprocess
import sys
from datetime import timedelta

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q) -> None:
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        local = [1.0 + rank, 10.0 - rank]          # rank 0: [1, 10]; rank 1: [2, 9]
        got = bench.max_over_ranks(local, world, torch.device("cpu"))
        rate = bench.job_rate(world, 5, 2.0, got[0])
        dist.barrier()
        q.put((rank, got, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_on_two_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, rate in results:
        assert got == [2.0, 10.0], (rank, got)                 # the slowest rank's times
        assert rate == pytest.approx(2 * 5 * 2.0 / 2.0e-3)      # both ranks' work / max time


def test_single_rank_is_unchanged():
    import torch
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.5, 4.0], 1, torch.device("cpu")) == [3.5, 4.0]
    assert bench.job_rate(1, 10, 3.0, 2.0) == pytest.approx(10 * 3.0 / 2.0e-3)


def _reference_arm(rank: int):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
               MASTER_ADDR="127.0.0.1")
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--gpus", "2", "--steps", "1", "--warmup", "3"],
                          capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)


def test_reference_arm_runs_on_rank_zero_only():
    r1 = _reference_arm(1)
    assert r1.returncode == 0 and r1.stdout.strip() == "", r1.stdout + r1.stderr
    r0 = _reference_arm(0)
    assert r0.returncode == 0, r0.stderr
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert "N=32768" in line["config"]["workload"]          # the headline workload
