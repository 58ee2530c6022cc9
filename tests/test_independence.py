"""The oracle and the CUDA path share nothing, and the product path never
reaches the oracle: checked on the sources (no GPU).

* oracle/ imports numpy and its own modules only (no torch, no ctypes, no
  package, no input generators, no benchmark);
* the package imports neither the oracle nor the input generators, and no CUDA
  source or header names the oracle;
* bench.py imports the oracle only inside the process that times the CPU
  baseline, and nothing committed reads the working folder."""

import ast
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "int4_kv_cache_paged_b200")


def _imports(path):
    """Absolute module names a Python file imports, with the top-level function each import sits in."""
    tree = ast.parse(open(path).read())
    found = []
    for top in tree.body:
        where = top.name if isinstance(top, (ast.FunctionDef, ast.ClassDef)) else None
        for n in ast.walk(top):
            if isinstance(n, ast.Import):
                found += [(a.name.split(".")[0], where) for a in n.names]
            elif isinstance(n, ast.ImportFrom) and n.level == 0:
                found.append((n.module.split(".")[0], where))
    return found


def test_oracle_imports_numpy_and_itself_only():
    files = glob.glob(os.path.join(ROOT, "oracle", "*.py"))
    assert files
    for f in files:
        assert {m for m, _ in _imports(f)} <= {"numpy"}, f


def test_package_never_reaches_the_oracle():
    for f in glob.glob(os.path.join(PKG, "*.py")):
        mods = {m for m, _ in _imports(f)}
        assert not mods & {"oracle", "workloads", "bench", "tests", "kvhelpers"}, f
    for f in glob.glob(os.path.join(PKG, "csrc", "*")) + glob.glob(os.path.join(ROOT, "include", "*")):
        assert "oracle" not in open(f, errors="replace").read().lower(), f


def test_bench_imports_the_oracle_only_in_its_cpu_baseline_process():
    where = {w for m, w in _imports(os.path.join(ROOT, "bench.py")) if m == "oracle"}
    assert where == {"_oracle_proc"}


def test_nothing_committed_reads_the_working_folder():
    paths = ([os.path.join(ROOT, "bench.py"), os.path.join(ROOT, "__graft_entry__.py")]
             + glob.glob(os.path.join(PKG, "*.py")) + glob.glob(os.path.join(PKG, "csrc", "*"))
             + glob.glob(os.path.join(ROOT, "oracle", "*.py")) + glob.glob(os.path.join(ROOT, "workloads", "*.py"))
             + glob.glob(os.path.join(ROOT, "include", "*")))
    for f in paths:
        assert not re.search(r"""(^|[\s"'/(])_work([/"')]|$)""", open(f, errors="replace").read(), re.M), f
