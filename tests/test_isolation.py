"""The oracle and the CUDA path stay apart (no GPU needed).

* Nothing in the product package imports ``oracle``, and the oracle imports nothing from the package.
* The CUDA sources include nothing from ``oracle/`` or ``workloads/``.
* In ``bench.py`` only the CPU-baseline / reference-arm functions reach the oracle.
* The shared input generators hold no arithmetic of the method: they import neither side.
"""
import ast
import glob
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sparse_attention_sum_b200")


def _imports(path):
    tree = ast.parse(open(path).read(), path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module:
            names.add(node.module)
    return names


def test_package_never_imports_the_oracle():
    files = glob.glob(os.path.join(PKG, "**", "*.py"), recursive=True)
    assert files
    for f in files:
        bad = {n for n in _imports(f) if n.split(".")[0] == "oracle"}
        assert not bad, f"{f} imports {bad}"


def test_oracle_and_generators_never_import_the_package():
    for f in glob.glob(os.path.join(ROOT, "oracle", "*.py")):
        bad = {n for n in _imports(f) if n.split(".")[0] == "sparse_attention_sum_b200"}
        assert not bad, f"{f} imports {bad}"
    for f in glob.glob(os.path.join(ROOT, "workloads", "*.py")):
        bad = {n for n in _imports(f) if n.split(".")[0] in ("sparse_attention_sum_b200", "oracle")}
        assert not bad, f"{f} imports {bad}"


def test_cuda_sources_include_nothing_from_the_oracle():
    for f in glob.glob(os.path.join(PKG, "csrc", "*")) + glob.glob(os.path.join(ROOT, "include", "*")):
        for line in open(f, errors="replace"):
            if line.lstrip().startswith("#include"):
                assert "oracle" not in line and "workloads" not in line, f"{f}: {line.strip()}"


def test_bench_reaches_the_oracle_only_from_its_cpu_arms():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    users = set()
    for fn in [n for n in ast.walk(tree) if isinstance(n, ast.FunctionDef)]:
        for node in ast.walk(fn):
            if isinstance(node, ast.ImportFrom) and node.module and node.module.startswith("oracle"):
                users.add(fn.name)
            if isinstance(node, ast.Import) and any(a.name.startswith("oracle") for a in node.names):
                users.add(fn.name)
    top = {n.module for n in tree.body if isinstance(n, ast.ImportFrom) and n.module}
    assert not any(m.startswith("oracle") for m in top), "bench.py imports the oracle at module level"
    assert users == {"oracle_rows", "oracle_kpool_rows"}, users
    # the oracle row functions are called only by the CPU arms, or handed to cpu_baseline as its row_fn
    allowed = {"cpu_baseline", "run_reference"}
    for fn in [n for n in ast.walk(tree) if isinstance(n, ast.FunctionDef)]:
        as_row_fn = set()
        for node in ast.walk(fn):
            if isinstance(node, ast.Call) and getattr(node.func, "id", None) == "cpu_baseline":
                as_row_fn |= {id(k.value) for k in node.keywords if k.arg == "row_fn"}
        for node in ast.walk(fn):
            if isinstance(node, ast.Name) and node.id in users and fn.name not in users:
                assert fn.name in allowed or id(node) in as_row_fn, f"{fn.name} reaches {node.id}"
