"""Static checks that the oracle and the CUDA path stay independent: the
product package (binding, build script, kernels) never imports the oracle,
the oracle never imports the product package, and the two share no source
file.  Only the seeded input generator (no arithmetic of the method) serves
both sides."""
from __future__ import annotations

import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "gated_delta_rule_66_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _files(top, exts):
    for d, dirs, names in os.walk(top):
        dirs[:] = [x for x in dirs if not x.startswith(("_build", "__pycache__"))]
        for n in names:
            if n.endswith(exts):
                yield os.path.join(d, n)


def _imported_modules(path):
    mods = set()
    for node in ast.walk(ast.parse(open(path).read(), path)):
        if isinstance(node, ast.Import):
            mods.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            if node.level == 0 and node.module:
                mods.add(node.module.split(".")[0])
    return mods


def test_product_package_never_imports_the_oracle():
    for path in _files(PKG, (".py",)):
        assert "oracle" not in _imported_modules(path), path


def test_kernels_reference_no_oracle_source():
    for path in _files(os.path.join(PKG, "csrc"), (".cu", ".cuh", ".h", ".cpp")):
        text = open(path).read()
        assert "oracle/" not in text and "#include \"../../oracle" not in text, path


def test_oracle_never_imports_the_product_package():
    for path in _files(ORACLE, (".py",)):
        mods = _imported_modules(path)
        assert "gated_delta_rule_66_b200" not in mods, path
        assert "torch" not in mods, path  # plain numpy / fractions only


def test_bench_imports_the_oracle_only_inside_the_cpu_baseline_leg():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    for node in tree.body:  # no module-level import of the oracle
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            names = [a.name for a in node.names] + [getattr(node, "module", None) or ""]
            assert not any(n.split(".")[0] == "oracle" for n in names)
    users = set()
    for fn in ast.walk(tree):
        if isinstance(fn, ast.FunctionDef):
            for node in ast.walk(fn):
                if isinstance(node, ast.Import) and any(a.name == "oracle" for a in node.names):
                    users.add(fn.name)
    assert users and users <= {"_oracle_head", "_warm"}, users
