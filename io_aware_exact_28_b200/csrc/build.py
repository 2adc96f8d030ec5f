"""Build libfa_b200.so in place with nvcc for sm_100a (no GPU needed to compile).

Usage: python io_aware_exact_28_b200/csrc/build.py [--verbose]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
ROOT = os.path.dirname(PKG)
OUT = os.path.join(PKG, "libfa_b200.so")
SOURCES = [os.path.join(HERE, "fa_api.cu")]
DEPS = SOURCES + [os.path.join(HERE, f) for f in ("sm100.cuh", "fwd_kernel.cuh", "bwd_kernel.cuh", "decode_kernel.cuh", "decode_tc_kernel.cuh")] \
    + [os.path.join(ROOT, "include", "fa.h"), os.path.abspath(__file__)]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(verbose: bool = False, out: str = OUT, defines=()) -> list[str]:
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-I", os.path.join(ROOT, "include"), "-I", HERE, "-o", out] + \
        [f"-D{d}" for d in defines] + SOURCES + ["-cudart", "static"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(p) <= t for p in DEPS)


def build(force: bool = False, verbose: bool = False, out: str = OUT, defines=()) -> str:
    """Compile (if stale) to `out`; `defines` (e.g. "FA_SOFTMAX_F32X2=0") build a variant."""
    if force or verbose or out != OUT or defines or not up_to_date():
        proc = subprocess.run(command(verbose, out, defines), capture_output=True, text=True)
        if proc.returncode != 0:
            raise RuntimeError(f"nvcc failed ({proc.returncode}):\n{proc.stdout}\n{proc.stderr}")
        if verbose:
            sys.stderr.write(proc.stderr)
    return out


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
