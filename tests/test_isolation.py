"""The product path and the oracle stay apart, and the product has no CPU fallback.

Static checks over the sources (import statements read with ``ast``) and one
subprocess that points the binding at a missing library.  No GPU needed.
"""
import ast
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "long_context_memory_b200")


def _imports(path):
    """(module name, enclosing function or None) of every import in a file."""
    tree = ast.parse(open(path, encoding="utf-8").read(), filename=path)
    found = []

    def walk(node, func):
        for ch in ast.iter_child_nodes(node):
            f = ch.name if isinstance(ch, (ast.FunctionDef, ast.AsyncFunctionDef)) else func
            if isinstance(ch, ast.Import):
                found.extend((a.name, f) for a in ch.names)
            elif isinstance(ch, ast.ImportFrom):
                found.append((("." * ch.level) + (ch.module or ""), f))
            elif isinstance(ch, ast.Call) and getattr(ch.func, "attr", getattr(ch.func, "id", "")) in (
                    "import_module", "__import__"):
                for a in ch.args:
                    if isinstance(a, ast.Constant) and isinstance(a.value, str):
                        found.append((a.value, f))
            walk(ch, f)

    walk(tree, None)
    return found


def _py_files(d):
    return [os.path.join(d, f) for f in sorted(os.listdir(d)) if f.endswith(".py")]


def test_product_package_never_imports_the_oracle():
    for path in _py_files(PKG):
        for mod, _ in _imports(path):
            assert mod.split(".")[0] != "oracle", f"{os.path.basename(path)} imports {mod}"


def test_oracle_imports_nothing_from_the_product():
    for path in _py_files(os.path.join(ROOT, "oracle")):
        for mod, _ in _imports(path):
            top = mod.lstrip(".").split(".")[0]
            assert top in ("", "math", "numpy", "msa_oracle", "__future__"), f"{os.path.basename(path)} imports {mod}"


def test_bench_runs_the_oracle_only_in_its_baseline_leg():
    # the cpu_baseline leg and --impl reference both go through time_oracle (and its pool worker,
    # time_oracle_shard)
    hits = [(m, f) for m, f in _imports(os.path.join(ROOT, "bench.py")) if m.split(".")[0] == "oracle"]
    assert hits, "bench.py no longer times the oracle"
    assert all(f in ("time_oracle", "time_oracle_shard") for _, f in hits), hits


def test_no_oracle_sources_in_the_cuda_build():
    # the library is built from the package's csrc only; no oracle file is compiled or included
    csrc = os.path.join(PKG, "csrc")
    for f in sorted(os.listdir(csrc)):
        text = open(os.path.join(csrc, f), encoding="utf-8").read()
        assert "oracle" not in text.lower(), f
    assert "oracle" not in open(os.path.join(PKG, "build.py"), encoding="utf-8").read()


def test_missing_library_raises_on_first_call():
    code = (
        "import long_context_memory_b200 as m\n"
        "m.LIB_PATH = '/nonexistent/libmsa.so'\n"
        "try:\n"
        "    m.chunk_offsets([0, 10, 300])\n"
        "except ImportError as e:\n"
        "    print('raised:', 'no CPU fallback' in str(e))\n"
        "else:\n"
        "    print('no error')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "raised: True", r.stdout + r.stderr
