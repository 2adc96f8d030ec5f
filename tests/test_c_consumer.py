"""Builds tests/c/abi_consumer.c, a plain C99 program, against include/fa.h with gcc
(-std=c99 -pedantic -Wall -Wextra -Werror), and the same source as C++17 with g++ (the
header's extern "C" block), links each to the built libfa_b200.so and runs it. CPU only:
the program makes host-side calls that return before any CUDA call."""
import os
import shutil
import subprocess

import pytest

import io_aware_exact_28_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("compiler,lang", [("gcc", ["-std=c99"]), ("g++", ["-x", "c++", "-std=c++17"])])
def test_c_program_builds_links_and_passes(tmp_path, compiler, lang):
    if shutil.which(compiler) is None:
        pytest.skip(f"needs {compiler}")
    fa.lib()                                   # the library exists and loads
    libdir = os.path.dirname(os.path.abspath(fa.LIB_PATH))
    exe = tmp_path / "abi_consumer"
    build = subprocess.run(
        [compiler, *lang, "-pedantic", "-Wall", "-Wextra", "-Werror",
         "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_consumer.c"),
         "-x", "none", "-L", libdir, "-lfa_b200", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
        capture_output=True, text=True, timeout=300)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "all checks passed" in run.stdout
