"""The product path has no CPU fallback and never touches the oracle: the
package, its CUDA sources and bench.py's native leg import nothing from
oracle/ (only the cpu_baseline / reference-arm sample classes of bench.py
do), and a missing library is an error, not a silent substitute."""
import ast
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_discrete_diffusion_denoise_b200")


INCLUDE_ORACLE = re.compile(r'#\s*include\s*[<"][^>"]*oracle')


def _oracle_imports(tree):
    """(enclosing function or class names, line) of every import of oracle."""
    out = []

    def visit(node, scope):
        for child in ast.iter_child_nodes(node):
            s = scope
            if isinstance(child, (ast.FunctionDef, ast.ClassDef)):
                s = scope + (child.name,)
            if isinstance(child, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in child.names):
                out.append((s, child.lineno))
            if isinstance(child, ast.ImportFrom) and (child.module or "").split(".")[0] == "oracle":
                out.append((s, child.lineno))
            visit(child, s)
    visit(tree, ())
    return out


def test_package_and_native_bench_never_import_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            p = os.path.join(dirpath, f)
            if f.endswith(".py"):
                assert _oracle_imports(ast.parse(open(p).read())) == [], p
            if f.endswith((".cu", ".cuh", ".h")):
                assert not INCLUDE_ORACLE.search(open(p).read()), p
    assert not INCLUDE_ORACLE.search(open(os.path.join(ROOT, "include", "dg.h")).read())
    sites = _oracle_imports(ast.parse(open(os.path.join(ROOT, "bench.py")).read()))
    assert sites, "bench.py's cpu_baseline leg times the oracle"
    for scope, line in sites:
        assert scope[:1] in (("OracleSample",), ("OracleFullStep",)), (scope, line)


def test_a_missing_library_is_an_error():
    code = ("import block_discrete_diffusion_denoise_b200 as d\n"
            "try:\n    d.load_library()\nexcept RuntimeError as e:\n    print('refused', 'not built' in str(e))\n")
    env = dict(os.environ, DG_LIBRARY=os.path.join(ROOT, "no_such_dir", "libdg.so"), PYTHONPATH=ROOT)
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    assert res.stdout.strip() == "refused True"


@pytest.mark.parametrize("name", ["smoke"])
def test_smoke_needs_a_device(name):
    """smoke() runs the CUDA path only: without a device it stops at its
    assertion instead of running anything on the host."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    import __graft_entry__ as g
    with pytest.raises(AssertionError):
        getattr(g, name)()
