"""Static checks that the product path and the oracle stay apart: the library and its
binding never reference the oracle, the oracle never reaches into the CUDA path, the
bench touches the oracle only in its CPU-baseline / reference legs, and a missing library
is an error, never a fallback."""
import ast
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_sparse_top_mean_b200")


def _files(top, exts):
    for d, _, fs in os.walk(top):
        for f in fs:
            if f.endswith(exts):
                yield os.path.join(d, f)


def test_library_and_binding_never_reference_the_oracle():
    for path in _files(PKG, (".py", ".cu", ".cuh", ".h")):
        src = open(path).read()
        assert not re.search(r"\boracle\b", src), path
        assert "parity_util" not in src, path


def test_oracle_never_reaches_into_the_cuda_path():
    for path in _files(os.path.join(ROOT, "oracle"), (".py",)):
        src = open(path).read()
        assert "block_sparse_top_mean_b200" not in src, path
        assert "csrc" not in src and "libmsa" not in src, path


def test_bench_uses_the_oracle_only_in_its_cpu_legs():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    allowed = re.compile(r"^(_w_(pool|prefill|decode)|run_reference\w*)$")
    for node in ast.walk(tree):
        if isinstance(node, ast.FunctionDef):
            for sub in ast.walk(node):
                names = []
                if isinstance(sub, ast.Import):
                    names = [a.name for a in sub.names]
                elif isinstance(sub, ast.ImportFrom):
                    names = [sub.module or ""]
                if any(n.split(".")[0] in ("oracle", "parity_util") for n in names):
                    assert allowed.match(node.name), node.name
    # and nothing at module level
    for node in tree.body:
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            names = [a.name for a in node.names] if isinstance(node, ast.Import) \
                else [node.module or ""]
            assert not any(n.split(".")[0] in ("oracle", "parity_util") for n in names)


def test_missing_library_is_an_error():
    code = ("from block_sparse_top_mean_b200 import _lib\n"
            "try:\n"
            "    _lib.load('/nonexistent/libmsa_b200.so')\n"
            "except ImportError:\n"
            "    print('raised')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.stdout.strip() == "raised", r.stdout + r.stderr
