"""The product path never reaches the oracle: the library package imports no
oracle module, bench.py imports it only inside its CPU legs (the
cpu_baseline sample and the reference arm), and the binding refuses to run
without the compiled library instead of falling back to anything."""
import ast
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _imports(tree):
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield node, a.name
        elif isinstance(node, ast.ImportFrom) and node.module:
            yield node, node.module


def test_package_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "dual_scale_solver_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            tree = ast.parse(open(os.path.join(pkg, fn)).read())
            names = [n for _, n in _imports(tree)]
            assert not any(n == "oracle" or n.startswith("oracle.") for n in names), fn


def test_bench_imports_the_oracle_only_in_its_cpu_legs():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    # the CPU legs: the oracle sample and the spawned workers that time the
    # oracle on every host core
    allowed = {"_oracle_sample", "_worker_init", "_worker_window", "_worker_iteration"}
    parents = {}
    for node in ast.walk(tree):
        for ch in ast.iter_child_nodes(node):
            parents[ch] = node
    for node, name in _imports(tree):
        if name == "oracle" or name.startswith("oracle."):
            p = node
            while p in parents and not isinstance(p, ast.FunctionDef):
                p = parents[p]
            assert isinstance(p, ast.FunctionDef) and p.name in allowed, p


def test_binding_refuses_to_run_without_the_library(monkeypatch, tmp_path):
    import dual_scale_solver_b200 as dq
    monkeypatch.setattr(dq, "_lib", None)
    monkeypatch.setattr(dq, "_LIB_PATH", str(tmp_path / "missing" / "libdq.so"))
    with pytest.raises(ImportError):
        dq.lib()
