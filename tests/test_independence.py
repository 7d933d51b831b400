"""The oracle and the CUDA path share no code, and the oracle stays test
infrastructure: the product package never reaches it, and the entry points
that may run it (smoke, the CPU baseline and the reference arm) import it
only inside those functions."""
import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "matrix_aware_optimizers_muon_b200")


def _files(top, exts):
    for dirpath, _dirs, names in os.walk(top):
        if "_build" in dirpath or "__pycache__" in dirpath:
            continue
        for nm in names:
            if nm.endswith(exts):
                yield os.path.join(dirpath, nm)


def _imported_modules(tree):
    """(module name, enclosing top-level function or None) for every import."""
    out = []
    for top in tree.body:
        scope = top.name if isinstance(top, (ast.FunctionDef, ast.AsyncFunctionDef)) else None
        for node in ast.walk(top):
            if isinstance(node, ast.Import):
                out += [(a.name, scope) for a in node.names]
            elif isinstance(node, ast.ImportFrom) and node.module:
                out.append((node.module, scope))
    return out


def test_product_sources_never_reach_the_oracle():
    for path in _files(PKG, (".py", ".cu", ".cuh", ".h")):
        with open(path, encoding="utf-8") as f:
            src = f.read()
        assert "oracle" not in src, path
    with open(os.path.join(ROOT, "include", "mo.h"), encoding="utf-8") as f:
        assert "oracle" not in f.read()


def test_oracle_and_workloads_import_no_product_code():
    for top, banned in (("oracle", ("matrix_aware_optimizers_muon_b200",)),
                        ("workloads", ("matrix_aware_optimizers_muon_b200", "oracle"))):
        for path in _files(os.path.join(ROOT, top), (".py",)):
            with open(path, encoding="utf-8") as f:
                tree = ast.parse(f.read())
            for mod, _scope in _imported_modules(tree):
                assert not mod.split(".")[0] in banned, (path, mod)


def test_oracle_imported_only_where_allowed():
    allowed = {"bench.py": {"cpu_baseline", "run_reference"}, "__graft_entry__.py": {"smoke"}}
    for name, scopes in allowed.items():
        with open(os.path.join(ROOT, name), encoding="utf-8") as f:
            tree = ast.parse(f.read())
        for mod, scope in _imported_modules(tree):
            if mod.split(".")[0] == "oracle":
                assert scope in scopes, (name, mod, scope)
