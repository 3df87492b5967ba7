"""The oracle and the CUDA path share nothing, and only test infrastructure reaches the
oracle: no file of the product package imports it or includes its C source, no file of
the oracle uses the product package or its CUDA sources, and bench.py imports the
oracle only inside the two functions that time it on the host (its CPU baseline and its
reference arm).  Nothing committed refers to the working directory `_work/`."""
import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "mxfp8_quantization_moe_mx_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _files(top, exts):
    for d, _, names in os.walk(top):
        for n in names:
            if n.endswith(exts):
                yield os.path.join(d, n)


def _imported_modules(tree):
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name.split(".")[0], node
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            yield node.module.split(".")[0], node


def test_product_package_never_reaches_the_oracle():
    for path in _files(PKG, (".py",)):
        tree = ast.parse(open(path).read())
        assert "oracle" not in {m for m, _ in _imported_modules(tree)}, path
    for path in _files(PKG, (".cu", ".cuh", ".h", ".c", ".cpp")):
        src = open(path).read()
        assert not re.search(r'#\s*include\s*[<"][^>"]*oracle', src), path


def test_oracle_never_uses_the_product():
    for path in _files(ORACLE, (".py",)):
        tree = ast.parse(open(path).read())
        assert "mxfp8_quantization_moe_mx_b200" not in {m for m, _ in _imported_modules(tree)}, path
    for path in _files(ORACLE, (".c", ".h")):
        src = open(path).read()
        assert "csrc" not in src and "mxq_device" not in src and "mxq_launch" not in src, path


def test_bench_imports_the_oracle_only_where_it_times_it():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    allowed = {"oracle_step_on_sample", "cpu_baseline"}
    for fn in [n for n in ast.walk(tree) if isinstance(n, (ast.FunctionDef, ast.AsyncFunctionDef))]:
        uses = [m for m, _ in _imported_modules(fn) if m == "oracle"]
        if uses:
            assert fn.name in allowed, fn.name
    top_level = [m for m, node in _imported_modules(ast.Module(body=tree.body, type_ignores=[]))
                 if node in tree.body and m == "oracle"]
    assert not top_level


def test_nothing_committed_refers_to_the_working_directory():
    skip = {os.path.join(ROOT, d) for d in ("_work", ".git", "gpurun_out", "baseline")}
    pat = re.compile(r"(^|[^A-Za-z0-9_])_work/")
    for d, dirs, names in os.walk(ROOT):
        dirs[:] = [x for x in dirs if os.path.join(d, x) not in skip and not x.startswith(".")]
        for n in names:
            path = os.path.join(d, n)
            if path == os.path.abspath(__file__):  # this check has to name the directory
                continue
            if n.endswith((".py", ".cu", ".cuh", ".h", ".c", ".sh", ".toml", ".cfg")):
                assert not pat.search(open(path, errors="replace").read()), path
