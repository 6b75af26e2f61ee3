"""The CUDA path and the oracle stay apart: the product never imports, links
or includes the oracle, the oracle includes nothing of the product, and the
only places that run the oracle are the test suite, smoke() and bench.py's
CPU-baseline and reference legs.  The binding also fails loudly without its
library (no CPU fallback)."""
import ast
import os
import re

import pytest

import block_sparse_attention_pa_b200 as pa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_sparse_attention_pa_b200")


def _imports_oracle(node) -> bool:
    if isinstance(node, ast.Import):
        return any(a.name.split(".")[0] == "oracle" for a in node.names)
    if isinstance(node, ast.ImportFrom):
        return (node.module or "").split(".")[0] == "oracle"
    return False


def _oracle_imports(path):
    """(import node, chain of enclosing nodes) for every import of oracle."""
    tree = ast.parse(open(path).read(), path)
    found = []

    def walk(node, chain):
        if _imports_oracle(node):
            found.append((node, chain))
        for child in ast.iter_child_nodes(node):
            walk(child, chain + [node])

    walk(tree, [])
    return found


def test_package_never_imports_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith(".py"):
                assert not _oracle_imports(os.path.join(dirpath, f)), f"{f} imports the oracle"


def test_native_sources_share_nothing():
    include = re.compile(r'^\s*#\s*include\s*[<"]([^>"]+)[>"]', re.M)
    product = [os.path.join(PKG, "csrc", f) for f in os.listdir(os.path.join(PKG, "csrc"))]
    product += [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))]
    for p in product:
        for inc in include.findall(open(p).read()):
            assert "oracle" not in inc, f"{p} includes {inc}"
    oracle_c = open(os.path.join(ROOT, "oracle", "pa_oracle.c")).read()
    # the oracle includes system headers only (angle brackets), none of the product's
    assert '#include "' not in oracle_c
    for inc in include.findall(oracle_c):
        assert inc.split("/")[0] not in ("pa.h", "sm100.cuh", "attn.cuh", "pool.cuh", "mask.cuh")
        assert not inc.endswith((".cuh", ".cu"))
    tree = ast.parse(open(os.path.join(ROOT, "oracle", "__init__.py")).read())
    for node in ast.walk(tree):
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            names = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module or ""]
            assert not any(n.startswith("block_sparse_attention_pa_b200") for n in names)


def test_bench_runs_the_oracle_only_in_its_cpu_legs():
    uses = _oracle_imports(os.path.join(ROOT, "bench.py"))
    assert uses, "bench.py has a CPU baseline and a reference arm, both timing the oracle"
    for node, chain in uses:
        funcs = [n.name for n in chain if isinstance(n, ast.FunctionDef)]
        assert funcs, "bench.py imports the oracle at module level"
        if funcs[-1] in ("oracle_estimate", "run_reference"):
            continue
        assert funcs[-1] == "main", f"oracle imported in {funcs[-1]}"
        guards = [ast.unparse(n.test) for n in chain if isinstance(n, ast.If)]
        assert any("no_cpu_baseline" in g for g in guards), "oracle reached outside the CPU-baseline leg"


def test_graft_entry_uses_the_oracle_only_to_build_and_check():
    for node, chain in _oracle_imports(os.path.join(ROOT, "__graft_entry__.py")):
        funcs = [n.name for n in chain if isinstance(n, ast.FunctionDef)]
        assert funcs and funcs[-1] in ("build", "smoke")


def test_binding_fails_loudly_without_its_library(monkeypatch, tmp_path):
    monkeypatch.setattr(pa, "LIB_PATH", str(tmp_path / "libpa.so"))
    monkeypatch.setattr(pa, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        pa.lib()
