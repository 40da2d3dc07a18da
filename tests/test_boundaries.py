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
    """The oracle (C++ and its Python marshalling) names neither the CUDA library nor torch,
    includes nothing of csrc/ or include/, and loads no shared library but its own."""
    for path in _files("oracle", (".py", ".c", ".cpp", ".h")):
        src = _text(path)
        for name in ("bit_group_quantized_fg_b200", "libfg", "torch", "fg.h", "csrc", "cuda"):
            assert name not in src, (path, name)
        if path.endswith(".py"):
            for m in re.finditer(r"CDLL\(([^)]*)\)", src):
                assert m.group(1).strip() == "path", (path, m.group(0))
            if "ctypes" in src:
                assert os.path.basename(path) in ("_lib.py", "decoder.py"), path
    lib_src = _text(os.path.join(ROOT, "oracle", "_lib.py"))
    assert 'LIB = os.path.join(HERE, "liboracle.so")' in lib_src
    for inc in re.findall(r'#include\s*[<"]([^>"]+)[>"]', _text(os.path.join(ROOT, "oracle", "fg_oracle.cpp"))):
        assert inc in ("cmath", "cstdint", "cstring", "vector", "omp.h"), inc


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
    allowed = {"__graft_entry__.py": {"smoke"}, "bench.py": {"oracle_sample", "cpu_baseline_line"}}
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


def test_oracle_build_flags_agree():
    """build() in __graft_entry__ compiles the oracle with the loader's flags (IEEE arithmetic,
    no contraction, no fast-math)."""
    import ast as _ast
    flags = []
    for path, name in ((os.path.join(ROOT, "__graft_entry__.py"), "ORACLE_FLAGS"),
                       (os.path.join(ROOT, "oracle", "_lib.py"), "FLAGS")):
        tree = _ast.parse(_text(path))
        vals = [_ast.literal_eval(n.value) for n in tree.body if isinstance(n, _ast.Assign)
                and any(isinstance(t, _ast.Name) and t.id == name for t in n.targets)]
        assert len(vals) == 1, (path, name)
        flags.append(vals[0])
    assert flags[0] == flags[1]
    assert "-ffp-contract=off" in flags[0] and "-fno-fast-math" in flags[0]
