"""The oracle and the CUDA path share no code, and the product never reaches the oracle.

Checked on the sources: nothing under sequence_all_re_b200/ (Python or CUDA)
imports, includes or loads anything under oracle/; nothing under oracle/
imports the product or includes its headers; the only module both sides'
tests use is synth/, which draws random numbers and holds no index arithmetic.
"""

import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def files_under(rel, exts):
    out = []
    for root, _, names in os.walk(os.path.join(ROOT, rel)):
        if "__pycache__" in root:
            continue
        out += [os.path.join(root, n) for n in names if n.endswith(exts)]
    return out


def python_imports(path):
    tree = ast.parse(open(path).read())
    mods = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            mods |= {a.name.split(".")[0] for a in node.names}
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            mods.add(node.module.split(".")[0])
    return mods


def test_product_never_imports_or_loads_the_oracle():
    for path in files_under("sequence_all_re_b200", (".py",)):
        assert "oracle" not in python_imports(path), path
        assert "libulysses_oracle" not in open(path).read(), path
    for path in files_under("sequence_all_re_b200", (".cu", ".cuh", ".h")):
        text = open(path).read()
        assert not re.search(r'#include\s+["<][^">]*oracle', text), path
        assert "oracle_ulysses" not in text, path


def test_oracle_never_uses_the_product():
    for path in files_under("oracle", (".py",)):
        assert not python_imports(path) & {"sequence_all_re_b200", "synth"}, path
    for path in files_under("oracle", (".c", ".h")):
        text = open(path).read()
        assert "ulysses_a2a.h" not in text and "ua2a" not in text, path


def test_synth_holds_no_index_arithmetic_of_the_method():
    # the shared input module draws numbers (and names slab shapes); it never
    # moves elements between layouts, so no call there re-lays out data
    relayout = {"permute", "transpose", "gather", "index_select", "scatter", "movedim",
                "as_strided", "unfold"}
    for path in files_under("synth", (".py",)):
        assert not python_imports(path) & {"oracle", "sequence_all_re_b200"}, path
        for node in ast.walk(ast.parse(open(path).read())):
            if isinstance(node, ast.Call) and isinstance(node.func, ast.Attribute):
                assert node.func.attr not in relayout, (path, node.func.attr)


def test_bench_reaches_the_oracle_only_in_its_baseline_legs():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    users = set()
    for fn in ast.walk(tree):
        if isinstance(fn, ast.FunctionDef):
            for node in ast.walk(fn):
                if isinstance(node, (ast.Import, ast.ImportFrom)):
                    names = ([a.name for a in node.names] if isinstance(node, ast.Import)
                             else [node.module or ""])
                    if any(n.split(".")[0] == "oracle" for n in names):
                        users.add(fn.name)
    assert users == {"cpu_oracle_baseline", "run_reference"}, users
