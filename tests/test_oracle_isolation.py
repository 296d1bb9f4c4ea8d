"""The oracle is test infrastructure: the library package never imports it, the oracle never
imports the library, and the benchmark runs it only in its CPU-baseline leg and its reference
arm (checked on the sources, CPU only)."""
import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "nvfp4_quantized_moe_group_b200")


def _imports(tree):
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            yield from (a.name for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module:
            yield node.module


def _py_files(top):
    for d, _, files in os.walk(top):
        yield from (os.path.join(d, f) for f in files if f.endswith(".py"))


def test_package_never_imports_the_oracle():
    for path in _py_files(PKG):
        with open(path) as f:
            src = f.read()
        assert "oracle" not in {m.split(".")[0] for m in _imports(ast.parse(src))}, path


def test_native_sources_never_mention_the_oracle():
    csrc = os.path.join(PKG, "csrc")
    for name in os.listdir(csrc):
        with open(os.path.join(csrc, name), errors="replace") as f:
            assert "oracle" not in f.read().lower(), name


def test_oracle_never_imports_the_library():
    for path in _py_files(os.path.join(ROOT, "oracle")):
        with open(path) as f:
            mods = {m.split(".")[0] for m in _imports(ast.parse(f.read()))}
        assert not mods & {"nvfp4_quantized_moe_group_b200", "torch", "workloads"}, (path, mods)


def test_bench_runs_the_oracle_only_in_its_baseline_legs():
    with open(os.path.join(ROOT, "bench.py")) as f:
        tree = ast.parse(f.read())
    users = set()
    for fn in ast.walk(tree):
        if isinstance(fn, ast.FunctionDef) and "oracle" in {m.split(".")[0] for m in _imports(fn)}:
            users.add(fn.name)
    assert users == {"_oracle_experts", "cpu_baseline_oracle", "run_reference"}, users
    assert "oracle" not in {m.split(".")[0] for m in _imports(ast.Module(body=[
        n for n in tree.body if not isinstance(n, ast.FunctionDef)], type_ignores=[]))}
