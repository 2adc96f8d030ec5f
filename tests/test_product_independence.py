"""The product path and the oracle are independent, and the product has no fallback.

* No file of the package (Python binding, CUDA sources, headers) imports, includes or
  names the oracle, and importing the package loads no oracle module.
* No oracle file imports the package or its compiled library.
* The seeded input generators (`workloads/`), the one module both sides use, import
  neither of them.
* With its shared library missing, the binding raises `FALibraryError` on first use:
  there is no CPU path to fall back to.
* Outside the tests, the oracle is imported only by `smoke()` of the entry module and by
  the CPU timing functions of `bench.py` (the CPU baseline and the reference arm).
CPU only.
"""
import ast
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "io_aware_exact_28_b200")


def _files(top, exts):
    for dirpath, _, names in os.walk(top):
        if "__pycache__" in dirpath:
            continue
        for n in names:
            if n.endswith(exts):
                yield os.path.join(dirpath, n)


def _imported_roots(path):
    """Top-level module names a Python file imports (absolute imports only)."""
    with open(path, encoding="utf-8") as f:
        tree = ast.parse(f.read(), path)
    roots = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            roots.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.level == 0 and node.module:
            roots.add(node.module.split(".")[0])
    return roots


def test_package_sources_never_reach_the_oracle():
    py = list(_files(PKG, (".py",)))
    assert py
    for p in py:
        assert "oracle" not in _imported_roots(p), p
    native = list(_files(PKG, (".cu", ".cuh", ".h", ".cpp"))) + \
        list(_files(os.path.join(ROOT, "include"), (".h",)))
    assert native
    for p in native:
        with open(p, encoding="utf-8") as f:
            src = f.read()
        assert not re.search(r'#\s*include\s*[<"][^>"]*oracle', src), p


def test_oracle_never_imports_the_package():
    files = list(_files(os.path.join(ROOT, "oracle"), (".py",)))
    assert files
    for p in files:
        roots = _imported_roots(p)
        assert "io_aware_exact_28_b200" not in roots and "ctypes" not in roots, p
        with open(p, encoding="utf-8") as f:
            assert "libfa_b200" not in f.read(), p


def test_input_generators_import_neither_side():
    files = list(_files(os.path.join(ROOT, "workloads"), (".py",)))
    assert files
    for p in files:
        roots = _imported_roots(p)
        assert not roots & {"oracle", "io_aware_exact_28_b200"}, (p, roots)


def _run(code, **env):
    e = dict(os.environ, **env)
    e["PYTHONPATH"] = ROOT + os.pathsep + e.get("PYTHONPATH", "")
    return subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                          cwd=ROOT, env=e, timeout=300)


def test_importing_the_package_loads_no_oracle_module():
    r = _run("import sys, io_aware_exact_28_b200 as fa\n"
             "fa.lib()\n"
             "bad = [m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')]\n"
             "print('LOADED', bad)\n")
    assert r.returncode == 0, r.stderr
    assert "LOADED []" in r.stdout, r.stdout


def test_missing_library_fails_loudly():
    missing = os.path.join(ROOT, "io_aware_exact_28_b200", "no_such_dir", "libfa_b200.so")
    r = _run("import io_aware_exact_28_b200 as fa\n"
             "try:\n"
             "    fa.lib()\n"
             "except fa.FALibraryError as e:\n"
             "    print('RAISED', type(e).__name__)\n"
             "else:\n"
             "    print('LOADED')\n", FA_B200_LIB=missing)
    assert r.returncode == 0, r.stderr
    assert "RAISED FALibraryError" in r.stdout, r.stdout


def _oracle_imports_by_function(path):
    """{enclosing top-level function name or '<module>': count} of oracle imports."""
    with open(path, encoding="utf-8") as f:
        tree = ast.parse(f.read(), path)
    found = {}

    def visit(node, owner):
        for child in ast.iter_child_nodes(node):
            name = owner
            if owner == "<module>" and isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)):
                name = child.name
            if isinstance(child, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in child.names):
                found[name] = found.get(name, 0) + 1
            if isinstance(child, ast.ImportFrom) and child.level == 0 and child.module and \
                    child.module.split(".")[0] == "oracle":
                found[name] = found.get(name, 0) + 1
            visit(child, name)
    visit(tree, "<module>")
    return found


def test_entry_points_reach_the_oracle_only_from_their_checking_legs():
    entry = _oracle_imports_by_function(os.path.join(ROOT, "__graft_entry__.py"))
    assert set(entry) == {"smoke"}, entry
    bench = _oracle_imports_by_function(os.path.join(ROOT, "bench.py"))
    assert bench and set(bench) <= {"oracle_rows_time", "oracle_baselines"}, bench


def test_bench_without_a_gpu_fails_instead_of_reporting():
    """On a machine without a GPU the benchmark's own arm exits non-zero and prints no
    result line: there is no CPU path that could stand in for the kernels."""
    import json
    import pytest
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; this checks the GPU-less case")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "1",
                        "--warmup", "3", "--no-cpu-baseline", "--no-e2e"],
                       capture_output=True, text=True, cwd=ROOT, timeout=300)
    assert r.returncode != 0
    for line in r.stdout.splitlines():
        try:
            obj = json.loads(line)
        except ValueError:
            continue
        assert "value" not in obj, line


def test_every_oracle_module_says_it_is_test_infrastructure():
    files = list(_files(os.path.join(ROOT, "oracle"), (".py",)))
    assert files
    for p in files:
        with open(p, encoding="utf-8") as f:
            doc = ast.get_docstring(ast.parse(f.read())) or ""
        assert "TEST INFRASTRUCTURE ONLY" in doc, p
