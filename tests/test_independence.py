"""The oracle and the product share no code, and the product never reaches
the oracle: checked on the sources (CPU only).

The oracle (``oracle/``) is test infrastructure; the product is the CUDA
library (``token_skipping_sparse_b200/csrc``, ``include/``) and its Python
binding.  Only the seeded input generators (``synthetic/``), which hold none
of the method's arithmetic, serve both sides.
"""

import ast
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _py_files(sub):
    out = []
    for dirpath, _, files in os.walk(os.path.join(ROOT, sub)):
        if "__pycache__" in dirpath:
            continue
        out += [os.path.join(dirpath, f) for f in files if f.endswith(".py")]
    return out


def _imported_modules(path):
    tree = ast.parse(open(path).read(), filename=path)
    mods = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            mods |= {a.name.split(".")[0] for a in node.names}
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            mods.add(node.module.split(".")[0])
    return mods


def test_product_and_generators_never_import_the_oracle():
    for path in _py_files("token_skipping_sparse_b200") + _py_files("synthetic"):
        assert "oracle" not in _imported_modules(path), path


def test_oracle_never_imports_the_product():
    for path in _py_files("oracle"):
        assert "token_skipping_sparse_b200" not in _imported_modules(path), path


def test_native_sources_do_not_name_the_oracle():
    for sub in ("token_skipping_sparse_b200/csrc", "include"):
        for dirpath, _, files in os.walk(os.path.join(ROOT, sub)):
            for f in files:
                if f.endswith((".cu", ".cuh", ".h", ".hpp", ".cpp")):
                    text = open(os.path.join(dirpath, f)).read()
                    assert "oracle" not in text.lower(), os.path.join(dirpath, f)


def test_importing_the_binding_loads_no_oracle_module():
    # a fresh interpreter: the binding loads libspts.so (built in-tree) and
    # must pull in nothing under oracle/
    code = ("import sys; sys.path.insert(0, %r)\n"
            "try:\n"
            "    import token_skipping_sparse_b200\n"
            "except ImportError as e:\n"
            "    print('SKIP', e); raise SystemExit(0)\n"
            "bad = [m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')]\n"
            "print('LOADED', bad)\n"
            "raise SystemExit(1 if bad else 0)\n") % ROOT
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr


def test_binding_without_the_library_fails_loudly(tmp_path):
    # the package copied without libspts.so: importing it raises, it does not
    # fall back to anything
    import shutil
    pkg = os.path.join(ROOT, "token_skipping_sparse_b200")
    dst = tmp_path / "token_skipping_sparse_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "__pycache__", "csrc"))
    code = ("import sys; sys.path.insert(0, %r)\n"
            "try:\n"
            "    import token_skipping_sparse_b200\n"
            "except ImportError as e:\n"
            "    print('RAISED', e); raise SystemExit(0)\n"
            "raise SystemExit(1)\n") % str(tmp_path)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "no CPU fallback" in r.stdout, r.stdout + r.stderr
