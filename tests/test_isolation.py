"""The product path and the oracle are independent: nothing in the package
(the binding, the build script, the CUDA sources and the C-ABI header)
imports, includes, links or loads anything under oracle/; the oracle
imports nothing from the package (the tests hand both sides the inputs of
the shared generator); and bench.py touches the oracle only inside its
CPU-baseline and reference-arm functions."""

import ast
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _py_imports(path):
    tree = ast.parse(open(path).read())
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module:
            names.add(node.module.split(".")[0])
    return names


def test_package_never_imports_the_oracle():
    for path in glob.glob(os.path.join(ROOT, "semi_markov_crf_b200", "*.py")):
        assert "oracle" not in _py_imports(path), path


def test_cuda_sources_and_header_never_reference_the_oracle():
    files = glob.glob(os.path.join(ROOT, "semi_markov_crf_b200", "csrc", "*")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))
    for path in files:
        text = open(path, errors="replace").read()
        assert not re.search(r"oracle", text, re.IGNORECASE), path


def test_oracle_uses_nothing_from_the_package():
    for path in glob.glob(os.path.join(ROOT, "oracle", "*.py")):
        assert "semi_markov_crf_b200" not in _py_imports(path), path
    src = open(os.path.join(ROOT, "oracle", "semicrf_oracle.c")).read()
    assert "semicrf.h" not in src and "csrc" not in src


def test_bench_uses_the_oracle_only_in_its_cpu_legs():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    users = set()
    for fn in [n for n in ast.walk(tree) if isinstance(n, ast.FunctionDef)]:
        for node in ast.walk(fn):
            if isinstance(node, (ast.Import, ast.ImportFrom)):
                mods = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module]
                if any(m and m.split(".")[0] == "oracle" for m in mods):
                    users.add(fn.name)
    # module level: no oracle import
    top = [n for n in tree.body if isinstance(n, (ast.Import, ast.ImportFrom))]
    for node in top:
        mods = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module]
        assert not any(m and m.split(".")[0] == "oracle" for m in mods)
    assert users <= {"oracle_sample_time", "cpu_baseline", "run_reference"}, users
