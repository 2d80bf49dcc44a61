"""The oracle and the CUDA path share no code (no GPU needed).

The product package never imports, includes or links anything under
oracle/, and the oracle never imports or includes the product package or its
CUDA sources; the only module both use is workloads/ (seeded random inputs,
none of the method's arithmetic).  bench.py reaches the oracle only inside
its CPU-timing functions."""
from __future__ import annotations

import ast
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _read(p):
    with open(p, encoding="utf-8") as f:
        return f.read()


def test_product_never_uses_the_oracle():
    pkg = os.path.join(ROOT, "mixed_precision_gemm_b200")
    for p in glob.glob(os.path.join(pkg, "**", "*.py"), recursive=True):
        for node in ast.walk(ast.parse(_read(p))):
            if isinstance(node, ast.Import):
                assert not any(a.name.split(".")[0] == "oracle" for a in node.names), p
            if isinstance(node, ast.ImportFrom):
                assert (node.module or "").split(".")[0] != "oracle", p
    for p in glob.glob(os.path.join(pkg, "csrc", "*")) + glob.glob(os.path.join(ROOT, "include", "*")):
        for inc in re.findall(r'#include\s*[<"]([^>"]+)[>"]', _read(p)):
            assert "oracle" not in inc, (p, inc)


def test_oracle_never_uses_the_product():
    for p in glob.glob(os.path.join(ROOT, "oracle", "*.py")):
        for node in ast.walk(ast.parse(_read(p))):
            names = [a.name for a in node.names] if isinstance(node, ast.Import) else \
                    [node.module or ""] if isinstance(node, ast.ImportFrom) else []
            assert not any(n.split(".")[0] == "mixed_precision_gemm_b200" for n in names), p
    for p in glob.glob(os.path.join(ROOT, "oracle", "*.c")) + glob.glob(os.path.join(ROOT, "oracle", "*.h")):
        for inc in re.findall(r'#include\s*[<"]([^>"]+)[>"]', _read(p)):
            assert inc in {"math.h", "stdint.h", "stdlib.h", "string.h", "omp.h", "stdio.h"}, (p, inc)


def test_workloads_import_neither_side():
    for p in glob.glob(os.path.join(ROOT, "workloads", "*.py")):
        for node in ast.walk(ast.parse(_read(p))):
            names = [a.name for a in node.names] if isinstance(node, ast.Import) else \
                    [node.module or ""] if isinstance(node, ast.ImportFrom) else []
            assert not any(n.split(".")[0] in ("oracle", "mixed_precision_gemm_b200") for n in names), p


def test_bench_imports_the_oracle_only_inside_cpu_timing():
    tree = ast.parse(_read(os.path.join(ROOT, "bench.py")))
    for node in tree.body:   # module level: no oracle import
        if isinstance(node, ast.Import):
            assert not any(a.name.split(".")[0] == "oracle" for a in node.names)
        if isinstance(node, ast.ImportFrom):
            assert (node.module or "").split(".")[0] != "oracle"
