"""The product path never touches the oracle, and fails loudly without its
CUDA library.

The oracle is test infrastructure: only the tests, the package smoke check
and the benchmark's CPU-baseline / reference legs may use it.  These checks
read the sources (no GPU): no file of the package imports or includes it;
bench.py imports it only inside its CPU legs; and a missing libep.so makes
the binding raise instead of computing anything on the CPU.
"""
import ast
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "combine_ep_layout_08_b200")


def test_package_sources_do_not_use_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for name in files:
            if not name.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                continue
            src = open(os.path.join(dirpath, name), encoding="utf-8").read()
            assert not re.search(r"^\s*(import|from)\s+oracle\b", src, re.M), name
            assert "ep_oracle" not in src, name
            assert not re.search(r'#include\s+["<][^">]*oracle', src), name


def test_bench_imports_the_oracle_only_in_its_cpu_legs():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py"), encoding="utf-8").read())
    allowed = {"oracle_sample", "oracle_timed_step", "cpu_baseline", "run_reference"}
    for fn in ast.walk(tree):
        if not isinstance(fn, ast.FunctionDef):
            continue
        for node in ast.walk(fn):
            names = []
            if isinstance(node, ast.Import):
                names = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                names = [node.module or ""]
            if any(n == "oracle" or n.startswith("oracle.") for n in names):
                assert fn.name in allowed, fn.name
    top = [n for n in tree.body if isinstance(n, (ast.Import, ast.ImportFrom))]
    for n in top:
        mods = [a.name for a in n.names] if isinstance(n, ast.Import) else [n.module or ""]
        assert "oracle" not in mods


def test_missing_library_raises(monkeypatch, tmp_path):
    import combine_ep_layout_08_b200 as ep

    monkeypatch.setattr(ep, "_lib", None)
    monkeypatch.setattr(ep, "_LIB_PATH", str(tmp_path / "libep.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback|There is no CPU fallback"):
        ep.load_library()
