"""The structure that the parity claims rest on, checked on the source text:

* the product package (block_sparse_long_exp_b200/) never imports the oracle,
  names it in code, or includes anything from it; the oracle imports nothing
  from the package (the two share no code);
* bench.py reaches the oracle only in its CPU-baseline and reference-arm
  functions, and __graft_entry__.py only in smoke();
* every GPU test file has a place in the run order of tests/conftest.py."""
import ast
import os
import re

import conftest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_sparse_long_exp_b200")


def _sources(top, exts):
    for dirpath, dirnames, files in os.walk(top):
        dirnames[:] = [d for d in dirnames if not d.startswith(("_build", "__pycache__", "."))]
        for f in sorted(files):
            if f.endswith(exts):
                yield os.path.join(dirpath, f)


def _imported(tree):
    """(module, node) for every import statement."""
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name, node
        elif isinstance(node, ast.ImportFrom) and node.module:
            yield node.module, node


def _docstrings(tree):
    out = set()
    for node in ast.walk(tree):
        if isinstance(node, (ast.Module, ast.FunctionDef, ast.AsyncFunctionDef, ast.ClassDef)):
            body = node.body
            if body and isinstance(body[0], ast.Expr) and isinstance(body[0].value, ast.Constant):
                out.add(id(body[0].value))
    return out


def test_product_package_never_reaches_the_oracle():
    checked = 0
    for path in _sources(PKG, (".py",)):
        tree = ast.parse(open(path, encoding="utf-8").read())
        for mod, _ in _imported(tree):
            assert mod.split(".")[0] != "oracle", f"{path} imports {mod}"
        docs = _docstrings(tree)
        for node in ast.walk(tree):
            if isinstance(node, ast.Constant) and isinstance(node.value, str) and id(node) not in docs:
                assert "oracle" not in node.value, f"{path} names the oracle in code: {node.value!r}"
        checked += 1
    for path in _sources(PKG, (".cu", ".cuh", ".h", ".cc", ".c")):
        text = open(path, encoding="utf-8").read()
        assert not re.search(r'#\s*include\s*[<"][^>"]*oracle', text), f"{path} includes the oracle"
        checked += 1
    assert checked >= 20


def test_oracle_shares_no_code_with_the_package():
    for path in _sources(os.path.join(ROOT, "oracle"), (".py",)):
        tree = ast.parse(open(path, encoding="utf-8").read())
        for mod, _ in _imported(tree):
            top = mod.split(".")[0]
            assert top in {"oracle", "numpy", "typing", "math", "__future__", "itertools"}, f"{path} imports {mod}"


def _oracle_importers(path):
    """Names of the functions that import the oracle (None: module level)."""
    tree = ast.parse(open(path, encoding="utf-8").read())
    owner = {}
    for fn in ast.walk(tree):
        if isinstance(fn, (ast.FunctionDef, ast.AsyncFunctionDef)):
            for node in ast.walk(fn):
                owner.setdefault(id(node), fn.name)
    return {owner.get(id(node)) for mod, node in _imported(tree) if mod.split(".")[0] == "oracle"}


def test_bench_and_entry_reach_the_oracle_only_where_allowed():
    assert _oracle_importers(os.path.join(ROOT, "bench.py")) <= {"cpu_oracle_rate", "run_reference"}
    assert _oracle_importers(os.path.join(ROOT, "__graft_entry__.py")) <= {"smoke"}


def test_every_gpu_test_file_has_a_place_in_the_run_order():
    tests = os.path.join(ROOT, "tests")
    mark = re.compile(r"^(pytestmark\s*=\s*pytest\.mark\.gpu\b|@pytest\.mark\.gpu\b)", re.M)
    gpu_files = sorted(f for f in os.listdir(tests) if f.startswith("test_") and f.endswith(".py")
                       and mark.search(open(os.path.join(tests, f), encoding="utf-8").read()))
    assert gpu_files and sorted(conftest.GPU_FILE_ORDER) == gpu_files
