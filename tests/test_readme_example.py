"""The Python example in README.md stays in step with the binding: it parses, and every
`fa.<name>(...)` call it makes names a public function of the package with keyword
arguments that function accepts. CPU only (the example itself needs a GPU)."""
import ast
import inspect
import os
import re

import io_aware_exact_28_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_example_matches_the_binding():
    with open(os.path.join(ROOT, "README.md"), encoding="utf-8") as f:
        blocks = re.findall(r"```python\n(.*?)```", f.read(), flags=re.S)
    assert blocks, "no python example in README.md"
    calls = 0
    for src in blocks:
        for node in ast.walk(ast.parse(src)):
            if isinstance(node, ast.Call) and isinstance(node.func, ast.Attribute) and \
                    isinstance(node.func.value, ast.Name) and node.func.value.id == "fa":
                fn = getattr(fa, node.func.attr, None)
                assert fn is not None and node.func.attr in fa.__all__, node.func.attr
                sig = inspect.signature(fn)
                bound = sig.bind_partial(*[None] * len(node.args),
                                         **{kw.arg: None for kw in node.keywords})
                assert bound is not None
                calls += 1
    assert calls >= 3
