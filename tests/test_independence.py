"""The oracle and the CUDA path share no code, and the product has no CPU fallback.

Checked from the sources, on the CPU:

* nothing under ``oracle/`` imports the library package, its build script or its
  kernels, and nothing in the package, its CUDA sources or the public header names the
  oracle;
* ``bench.py`` reaches the oracle only from its CPU-baseline helper (``oracle_sample``,
  used by the ``cpu_baseline`` leg and the reference arm);
* with ``libfvattn.so`` absent, every entry point of the binding raises instead of
  computing anything.
"""
import ast
import glob
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "free_adaptive_block_b200")


def imported_modules(path):
    """(module name, enclosing function or None) for every import in a Python file."""
    tree = ast.parse(open(path, encoding="utf-8").read(), path)
    out = []

    def visit(node, fn):
        for child in ast.iter_child_nodes(node):
            name = fn
            if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)):
                name = child.name
            if isinstance(child, ast.Import):
                out.extend((a.name, fn) for a in child.names)
            elif isinstance(child, ast.ImportFrom):
                base = "." * child.level + (child.module or "")
                out.append((base, fn))
                out.extend((f"{base}.{a.name}", fn) for a in child.names)
            visit(child, name)

    visit(tree, None)
    return out


def test_oracle_imports_nothing_of_the_library():
    files = glob.glob(os.path.join(ROOT, "oracle", "**", "*.py"), recursive=True)
    assert files
    for f in files:
        for mod, _ in imported_modules(f):
            assert not mod.startswith(("free_adaptive_block_b200", "_build", "ctypes", "torch")), (f, mod)
        text = open(f, encoding="utf-8").read()
        assert "libfvattn" not in text and "csrc" not in text, f


def test_library_and_kernels_never_name_the_oracle():
    for f in glob.glob(os.path.join(PKG, "**", "*.py"), recursive=True):
        for mod, _ in imported_modules(f):
            assert not mod.split(".")[0] == "oracle", (f, mod)
    sources = [f for f in glob.glob(os.path.join(PKG, "csrc", "*"))
               if f.endswith((".cu", ".cuh", ".h", ".cpp"))] + glob.glob(os.path.join(ROOT, "include", "*.h"))
    assert sources
    for f in sources:
        text = open(f, encoding="utf-8").read()
        assert "oracle" not in text.lower(), f


def test_bench_reaches_the_oracle_only_from_its_cpu_baseline_helper():
    uses = [(m, fn) for m, fn in imported_modules(os.path.join(ROOT, "bench.py"))
            if m.split(".")[0] == "oracle"]
    assert uses, "the CPU-baseline leg imports the oracle"
    assert {fn for _, fn in uses} == {"oracle_sample"}


def test_no_cpu_fallback_without_the_library(monkeypatch, tmp_path):
    import free_adaptive_block_b200 as fv
    monkeypatch.setattr(fv, "LIB_PATH", str(tmp_path / "libfvattn.so"))
    monkeypatch.setattr(fv, "_lib", None)
    g = fv.Geometry(1, 1, 1, 8, 16, 64, 1, 8, 16)
    calls = [
        lambda: fv.lib(),
        lambda: fv.fvattn_num_blocks(g),
        lambda: fv.fvattn_attn_workspace_size(g),
        lambda: fv.fvattn_route_workspace_size(g),
        lambda: fv.fvattn_num_sms(),
        lambda: fv.fvattn_status_string(0),
    ]
    for call in calls:
        with pytest.raises(RuntimeError, match="missing"):
            call()
