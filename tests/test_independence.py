"""The oracle and the CUDA path share no code: the package never imports the
oracle, the oracle never imports the package nor includes its headers, and
bench.py touches the oracle only in its CPU-baseline and reference legs."""
import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _imports(path):
    tree = ast.parse(open(path).read())
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module:
            names.add(node.module.split(".")[0])
    return names


def test_package_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "precision_label_chunk_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith(".py"):
                assert "oracle" not in _imports(os.path.join(dirpath, f)), f
            if f.endswith((".cu", ".cuh", ".h")):
                assert "oracle" not in open(os.path.join(dirpath, f)).read().lower(), f


def test_oracle_never_uses_the_package():
    odir = os.path.join(ROOT, "oracle")
    for f in os.listdir(odir):
        path = os.path.join(odir, f)
        if f.endswith(".py"):
            assert "precision_label_chunk_b200" not in _imports(path), f
        if f.endswith((".c", ".h")):
            text = open(path).read()
            includes = re.findall(r'^\s*#\s*include\s*(\S+)', text, flags=re.M)
            assert includes and all(i.startswith("<") for i in includes), f"{f}: {includes}"   # system headers only


def test_bench_uses_the_oracle_only_in_host_legs():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    legs = {"cpu_baseline", "run_reference", "run_reference_other", "run_topk", "run_kahan"}
    for fn in [n for n in tree.body if isinstance(n, ast.FunctionDef)]:
        uses = any(isinstance(n, (ast.Import, ast.ImportFrom)) and
                   any((a.name if isinstance(n, ast.Import) else n.module or "").startswith("oracle")
                       for a in (n.names if isinstance(n, ast.Import) else [n]))
                   for n in ast.walk(fn))
        if uses:
            assert fn.name in legs, f"bench.py:{fn.name} imports the oracle"
