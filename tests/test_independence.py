"""The oracle and the CUDA path share no code: no module of the package imports
the oracle, the oracle imports nothing of the package, and the oracle's C
source includes no header of the package (the seeded input generators in
workloads.py hold none of the method's arithmetic and serve both)."""
import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_scaled_precision_05_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _imports(path):
    tree = ast.parse(open(path).read(), filename=path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            names.add(node.module.split(".")[0])
    return names


def _files(top, ext):
    for d, _, fs in os.walk(top):
        if "_build" in d or "__pycache__" in d:
            continue
        for f in fs:
            if f.endswith(ext):
                yield os.path.join(d, f)


def test_package_does_not_import_the_oracle():
    for p in _files(PKG, ".py"):
        assert "oracle" not in _imports(p), p


def test_oracle_does_not_import_the_package():
    for p in _files(ORACLE, ".py"):
        assert "block_scaled_precision_05_b200" not in _imports(p), p


def test_oracle_c_includes_only_system_headers():
    for p in _files(ORACLE, ".c"):
        for inc in re.findall(r'^\s*#\s*include\s*([<"][^>"]+[>"])', open(p).read(), re.M):
            assert inc.startswith("<"), (p, inc)


def test_cuda_sources_include_nothing_of_the_oracle():
    for ext in (".cu", ".cuh", ".h"):
        for p in _files(PKG, ext):
            for inc in re.findall(r'^\s*#\s*include\s*([<"][^>"]+[>"])', open(p).read(), re.M):
                assert "oracle" not in inc, (p, inc)
