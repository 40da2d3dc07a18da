"""CPU checks of the separation between the product, the oracle and the input generator.

The CUDA library and its binding never reach the oracle (no CPU path stands in for a kernel);
the oracle never reaches the CUDA library; the seeded input generator depends on neither; and
outside tests/ only the smoke entry point and the benchmark's CPU-baseline leg import the
oracle, inside those functions."""
import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _files(sub, exts):
    out = []
    for dirpath, _, names in os.walk(os.path.join(ROOT, sub)):
        out += [os.path.join(dirpath, n) for n in names if n.endswith(exts)]
    return out


def _text(path):
    with open(path, encoding="utf-8", errors="replace") as f:
        return f.read()


def test_product_never_reaches_the_oracle():
    for path in _files("bit_group_quantized_fg_b200", (".py", ".cu", ".cuh", ".h")) + _files("include", (".h",)):
        assert not re.search(r"\boracle\b", _text(path)), path


def test_oracle_never_reaches_the_cuda_path():
    for path in _files("oracle", (".py", ".c", ".h")):
        src = _text(path)
        for name in ("bit_group_quantized_fg_b200", "libfg", "ctypes", "torch"):
            assert name not in src, (path, name)


def test_input_generator_depends_on_neither():
    for path in _files("fg_synth", (".py", ".cu")):
        src = _text(path)
        assert "bit_group_quantized_fg_b200" not in src and not re.search(r"^\s*(import|from) oracle", src, re.M), path


def _oracle_import_sites(path):
    """(enclosing function name or None) for every import of the oracle in a Python file."""
    tree = ast.parse(_text(path))
    sites = []

    def visit(node, fn):
        for child in ast.iter_child_nodes(node):
            inner = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else fn
            if isinstance(child, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in child.names):
                sites.append(fn)
            if isinstance(child, ast.ImportFrom) and (child.module or "").split(".")[0] == "oracle":
                sites.append(fn)
            visit(child, inner)

    visit(tree, None)
    return sites


def test_oracle_imported_only_by_tests_smoke_and_cpu_baseline():
    allowed = {"__graft_entry__.py": {"smoke"}, "bench.py": {"oracle_sample"}}
    for path in _files(".", (".py",)):
        rel = os.path.relpath(path, ROOT)
        top = rel.split(os.sep)[0]
        if top in ("tests", "oracle", "_work", "gpurun_out", "baseline") or top.startswith("."):
            continue
        sites = _oracle_import_sites(path)
        if not sites:
            continue
        assert rel in allowed, f"{rel} imports the oracle"
        assert set(sites) <= allowed[rel], (rel, sites)
