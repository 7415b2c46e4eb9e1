"""The oracle and the product path stay apart (CPU only, static checks).

* nothing in the package (its Python modules, CUDA / C sources and the ABI
  header) or in synthetic/ imports the oracle, and no native source names it;
* nothing in oracle/ or synthetic/ imports the package;
* bench.py imports the oracle only inside its CPU-oracle timing function and
  __graft_entry__ only inside smoke();
* the binding refuses to load without the compiled library (no fallback): a
  copy of the package without liblsq.so raises ImportError on import.
"""
import ast
import glob
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = "nf4_layer_streamed_blockwise_b200"


def _imports(path):
    """(imported module, enclosing function or None) for every import in a file."""
    tree = ast.parse(open(path).read(), filename=path)
    out = []

    def visit(node, fn):
        for child in ast.iter_child_nodes(node):
            name = fn
            if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)):
                name = child.name
            if isinstance(child, ast.Import):
                out.extend((a.name, name) for a in child.names)
            elif isinstance(child, ast.ImportFrom):
                mod = ("." * child.level) + (child.module or "")
                out.append((mod, name))
            visit(child, name)

    visit(tree, None)
    return out


def _py(*parts):
    return sorted(glob.glob(os.path.join(ROOT, *parts)))


def test_product_and_inputs_never_import_the_oracle():
    files = _py(PKG, "*.py") + _py("synthetic", "*.py")
    assert len(files) >= 6
    for f in files:
        for mod, _ in _imports(f):
            assert not mod.split(".")[0] == "oracle", f"{f} imports {mod}"


def test_native_sources_do_not_name_the_oracle():
    files = _py(PKG, "csrc", "*") + _py("include", "*.h")
    assert any(f.endswith(".cu") for f in files)
    for f in files:
        assert "oracle" not in open(f, errors="replace").read().lower(), f


def test_oracle_and_inputs_never_import_the_product():
    for f in _py("oracle", "*.py") + _py("synthetic", "*.py"):
        for mod, _ in _imports(f):
            assert not mod.split(".")[0] == PKG, f"{f} imports {mod}"


def test_bench_and_entry_use_the_oracle_only_in_their_cpu_legs():
    allowed = {"bench.py": {"oracle_sample"}, "__graft_entry__.py": {"smoke"}}
    for name, fns in allowed.items():
        uses = [(mod, fn) for mod, fn in _imports(os.path.join(ROOT, name)) if mod.split(".")[0] == "oracle"]
        assert uses, name
        for mod, fn in uses:
            assert fn in fns, f"{name}: oracle imported in {fn or 'module scope'}"


def test_binding_fails_loudly_without_the_library(tmp_path):
    dst = tmp_path / PKG
    dst.mkdir()
    for f in ("__init__.py", "lib.py"):
        shutil.copy(os.path.join(ROOT, PKG, f), dst / f)
    assert not (dst / "liblsq.so").exists()
    r = subprocess.run([sys.executable, "-c", f"import {PKG}.lib"], cwd=tmp_path, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "liblsq.so is missing" in r.stderr
