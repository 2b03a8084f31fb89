"""The oracle and the CUDA path share nothing, and the product has no other path, on the CPU.

The product (the package and its CUDA sources) never imports, includes or
names the oracle; the oracle imports nothing of the package; and bench.py
imports the oracle only inside its CPU-baseline and reference-arm functions,
never at module level, so its GPU arm cannot reach it. Without the built
library the binding raises on the first call that needs it."""
import ast
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sparse_long_sequence_dilated_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _files(top, exts):
    for d, _, names in os.walk(top):
        for n in names:
            if n.endswith(exts):
                yield os.path.join(d, n)


def test_product_modules_do_not_load_the_oracle():
    code = ("import sys\n"
            "import sparse_long_sequence_dilated_b200.dilattn, sparse_long_sequence_dilated_b200.seqpar\n"
            "import sparse_long_sequence_dilated_b200.flops, sparse_long_sequence_dilated_b200.workloads\n"
            "import sparse_long_sequence_dilated_b200.build\n"
            "print(sorted(m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')))\n")
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                         timeout=300)
    assert res.returncode == 0, res.stderr
    assert res.stdout.strip() == "[]"


def test_package_sources_never_name_the_oracle():
    for f in _files(PKG, (".py", ".cu", ".cuh", ".h")):
        text = open(f, encoding="utf-8").read()
        assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
        assert not re.search(r"#\s*include\s*[<\"][^>\"]*oracle", text), f
        assert "importlib" not in text or "oracle" not in text, f


def test_oracle_imports_nothing_of_the_package():
    for f in _files(ORACLE, (".py",)):
        tree = ast.parse(open(f, encoding="utf-8").read())
        for node in ast.walk(tree):
            if isinstance(node, ast.Import):
                names = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                names = [node.module or ""]
            else:
                continue
            for n in names:
                assert not n.startswith("sparse_long_sequence_dilated_b200"), (f, n)
                assert n.split(".")[0] in {"math", "typing", "numpy", "__future__", "dilated",
                                           ""}, (f, n)


def test_bench_imports_the_oracle_only_in_its_cpu_legs():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py"), encoding="utf-8").read())
    allowed = {"cpu_baseline", "_oracle_task", "run_reference"}
    for node in tree.body:  # module level: no oracle import
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            mods = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module]
            assert "oracle" not in mods
    found = set()
    for fn in ast.walk(tree):
        if isinstance(fn, ast.FunctionDef):
            for node in ast.walk(fn):
                if isinstance(node, ast.Import) and any(a.name == "oracle" for a in node.names):
                    found.add(fn.name)
                if isinstance(node, ast.ImportFrom) and node.module == "oracle":
                    found.add(fn.name)
    assert found and found <= allowed, found


def test_a_missing_library_fails_loudly(tmp_path):
    """With no built library there is no other path: a copy of the package's
    Python files without the library raises on the first call that needs it."""
    import shutil
    dst = tmp_path / "sparse_long_sequence_dilated_b200"
    dst.mkdir()
    for f in os.listdir(PKG):
        if f.endswith(".py"):
            shutil.copy(os.path.join(PKG, f), dst / f)
    code = (
        "from sparse_long_sequence_dilated_b200 import dilattn\n"
        "assert not dilattn.LIB_PATH.startswith(" + repr(ROOT) + ")\n"
        "for call in (lambda: dilattn.load(), lambda: dilattn.status_string(0),\n"
        "             lambda: dilattn.bwd_workspace_size(1, 64, 1, 64)):\n"
        "    try:\n"
        "        call()\n"
        "        print('no error')\n"
        "    except RuntimeError as e:\n"
        "        print('raised', 'is missing' in str(e))\n")
    env = dict(os.environ, PYTHONPATH=str(tmp_path))
    res = subprocess.run([sys.executable, "-c", code], cwd=str(tmp_path), env=env,
                         capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr
    assert res.stdout.split() == ["raised", "True"] * 3, res.stdout
