"""The product path never reaches the oracle (CPU only, static).

The oracle is test infrastructure.  The package (bindings, generator, build) and the CUDA sources must not
import, include or open anything under oracle/.  bench.py may call it only from its CPU-baseline helpers,
oracle_compress and oracle_decode, which the reference arm and the CPU baseline use.
"""
import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "residual_kv_cache_delta_b200")


def _imports_oracle(node) -> bool:
    if isinstance(node, ast.Import):
        return any(a.name == "oracle" or a.name.startswith("oracle.") for a in node.names)
    if isinstance(node, ast.ImportFrom):
        return node.module is not None and (node.module == "oracle" or node.module.startswith("oracle."))
    return False


def _py_files(top):
    for d, _, files in os.walk(top):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(d, f)


def test_package_never_imports_the_oracle():
    for path in _py_files(PKG):
        tree = ast.parse(open(path).read(), path)
        assert not any(_imports_oracle(n) for n in ast.walk(tree)), path
        assert "deltakv_oracle" not in open(path).read(), path


def test_cuda_sources_share_nothing_with_the_oracle():
    csrc = os.path.join(PKG, "csrc")
    for f in os.listdir(csrc):
        text = open(os.path.join(csrc, f), errors="replace").read()
        assert "oracle" not in text.lower(), f
    for f in os.listdir(os.path.join(ROOT, "include")):
        assert "oracle" not in open(os.path.join(ROOT, "include", f)).read().lower(), f


def test_bench_calls_the_oracle_only_from_its_cpu_baseline_helpers():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    allowed = {"oracle_compress", "oracle_decode"}
    assert not any(_imports_oracle(n) for n in tree.body), "module-level oracle import"
    for fn in (n for n in ast.walk(tree) if isinstance(n, (ast.FunctionDef, ast.AsyncFunctionDef))):
        direct = [n for n in ast.walk(fn) if _imports_oracle(n)]
        if direct:
            assert fn.name in allowed, f"{fn.name} imports the oracle"
