"""The product path has no fallback and never reaches the oracle.

* Importing the binding without the built library raises at once.
* No module of the package, and no CUDA/C++ source of the library, imports or
  includes anything from ``oracle/``.
* ``bench.py`` imports the oracle only inside the function that times it (the
  CPU baseline and the reference arm); the GPU arm's code has no import of it.
"""

import ast
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "mla_latent_kv_38_b200")


def _imports(tree):
    """(module name, enclosing function or None) for every import in `tree`."""
    out = []

    def visit(node, fn):
        for child in ast.iter_child_nodes(node):
            f = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else fn
            if isinstance(child, ast.Import):
                out.extend((a.name, fn) for a in child.names)
            elif isinstance(child, ast.ImportFrom):
                mod = child.module or ""
                out.append((mod, fn))
                out.extend((f"{mod}.{a.name}", fn) for a in child.names)
            visit(child, f)

    visit(tree, None)
    return out


def test_binding_import_fails_loudly_without_the_library():
    env = dict(os.environ, MLA_B200_LIB=os.path.join(ROOT, "no-such-dir", "libmla_b200.so"))
    code = ("import sys\n"
            "try:\n"
            "    import mla_latent_kv_38_b200.binding\n"
            "except ImportError as e:\n"
            "    print('raised:', e); sys.exit(0)\n"
            "sys.exit(3)\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "is missing" in r.stdout


def test_package_never_imports_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            path = os.path.join(dirpath, f)
            if f.endswith(".py"):
                tree = ast.parse(open(path).read(), path)
                for mod, _ in _imports(tree):
                    assert not mod.split(".")[0] == "oracle", (path, mod)
            elif f.endswith((".cu", ".cuh", ".h", ".cpp", ".c")):
                for line in open(path):
                    if line.lstrip().startswith("#include"):
                        assert "oracle" not in line, (path, line)


def test_bench_imports_the_oracle_only_where_it_times_it():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    sites = [fn for mod, fn in _imports(tree) if mod.split(".")[0] == "oracle"]
    assert sites, "the CPU baseline must time the oracle"
    assert set(sites) == {"oracle_sample_rate"}
