"""The oracle and the CUDA path stay apart (no GPU).

- No product file (the package's Python, CUDA sources and the ABI header) imports, includes
  or loads the oracle, and no oracle file names the package, its sources or its header.
- The input generators use neither side.
- bench.py reaches the oracle only from its CPU-baseline and reference legs, and the entry
  module only to build it and in its smoke check.
- The package fails loudly when its library has not been built: there is no fallback."""

import ast
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "long_context_compressed_layer_b200")


def _files(*patterns):
    out = []
    for p in patterns:
        out += glob.glob(os.path.join(ROOT, p), recursive=True)
    return sorted(f for f in out if "__pycache__" not in f)


def _hits(files, pattern):
    rx = re.compile(pattern)
    return [(os.path.relpath(f, ROOT), i + 1, line.strip())
            for f in files for i, line in enumerate(open(f, encoding="utf-8"))
            if rx.search(line)]


ORACLE_USE = r"\bimport oracle\b|\bfrom oracle\b|liboracle|csa_oracle|oracle/|oracle\.(cpp|h)\b"
PRODUCT_USE = (r"long_context_compressed_layer_b200|libcsa_b200|csrc|common\.cuh|"
               r"#include\s*[<\"][^>\"]*csa\.h")


def test_product_files_never_use_the_oracle():
    files = _files("long_context_compressed_layer_b200/**/*.py",
                   "long_context_compressed_layer_b200/csrc/*", "include/*.h")
    assert len(files) >= 10
    assert _hits(files, ORACLE_USE) == []


def test_oracle_files_never_use_the_product():
    files = _files("oracle/*.py", "oracle/*.cpp", "oracle/*.h", "oracle/*.c")
    assert any(f.endswith(".cpp") for f in files)
    assert _hits(files, PRODUCT_USE) == []


def test_input_generators_use_neither_side():
    files = _files("synth/*.py")
    assert files
    assert _hits(files, ORACLE_USE) == []
    assert _hits(files, r"\bimport long_context_compressed_layer_b200|"
                        r"\bfrom long_context_compressed_layer_b200") == []


def _enclosing_imports(tree):
    """(function name or None, the chain of `if` tests above it) for each import of the
    oracle module."""
    found = []

    def walk(node, fn, tests):
        for child in ast.iter_child_nodes(node):
            f, t = fn, tests
            if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)):
                f, t = child.name, []
            elif isinstance(child, ast.If):
                t = tests + [ast.unparse(child.test)]
            if isinstance(child, ast.Import) and any(a.name == "oracle" for a in child.names):
                found.append((fn, tests))
            if isinstance(child, ast.ImportFrom) and (child.module or "").startswith("oracle"):
                found.append((fn, tests))
            walk(child, f, t)

    walk(tree, None, [])
    return found


def test_bench_reaches_the_oracle_only_from_its_baseline_legs():
    with open(os.path.join(ROOT, "bench.py"), encoding="utf-8") as fh:
        tree = ast.parse(fh.read())
    uses = _enclosing_imports(tree)
    assert uses, "bench.py times the oracle somewhere"
    legs = {"prefill_cpu_baseline", "cpu_baseline_sample", "run_reference"}
    for fn, tests in uses:
        assert fn is not None, "the oracle is imported at module level"
        # the HCA line takes its CPU baseline inline, behind the baseline switch
        assert fn in legs or any("no_cpu_baseline" in t for t in tests), (fn, tests)


def test_the_package_fails_loudly_without_its_library(monkeypatch):
    import long_context_compressed_layer_b200 as csa

    monkeypatch.setattr(csa, "_lib", None)
    monkeypatch.setattr(csa, "LIB_PATH", os.path.join(ROOT, "no_such_dir", "libcsa_b200.so"))
    with pytest.raises(RuntimeError, match="is missing"):
        csa.lib()


def test_entry_module_uses_the_oracle_only_to_build_it_and_in_the_smoke_check():
    with open(os.path.join(ROOT, "__graft_entry__.py"), encoding="utf-8") as fh:
        uses = _enclosing_imports(ast.parse(fh.read()))
    assert uses and all(fn in ("build", "smoke") for fn, _ in uses), uses
