"""The oracle and the CUDA path stay apart, and the product has no fallback.

- Nothing in the package or in the input generators imports the oracle; `bench.py` and
  the entry points import it only inside the functions that time or check against it.
- The oracle imports nothing of the package and loads no shared library.
- The CUDA sources include nothing from the oracle, the input generators or the tests.
- Without its compiled library the binding refuses to import: there is no other
  implementation behind it.
"""
import ast
import importlib.util
import os
import re
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "decoder_only_transformer_int4_b200")


def _py_files(d):
    for name in sorted(os.listdir(d)):
        if name.endswith(".py"):
            yield os.path.join(d, name)


def _imports(path):
    """(imported module, enclosing top-level function or None) for every import."""
    tree = ast.parse(open(path).read(), path)
    out = []

    def visit(node, func):
        for child in ast.iter_child_nodes(node):
            f = func
            if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) and func is None:
                f = child.name
            if isinstance(child, ast.Import):
                out.extend((a.name, f) for a in child.names)
            elif isinstance(child, ast.ImportFrom):
                if child.level == 0 and child.module:
                    out.append((child.module, f))
            visit(child, f)

    visit(tree, None)
    return out


def _is_oracle(mod):
    return mod == "oracle" or mod.startswith("oracle.")


def test_package_and_input_generators_never_import_the_oracle():
    files = list(_py_files(PKG)) + list(_py_files(os.path.join(ROOT, "synth")))
    assert files
    for path in files:
        bad = [m for m, _ in _imports(path) if _is_oracle(m)]
        assert not bad, (path, bad)


@pytest.mark.parametrize("name,allowed", [
    ("bench.py", {"_oracle_sample", "run_reference"}),
    ("__graft_entry__.py", {"smoke"}),
])
def test_oracle_imported_only_where_it_is_timed_or_checked(name, allowed):
    users = {f for m, f in _imports(os.path.join(ROOT, name)) if _is_oracle(m)}
    assert users, name
    assert users <= allowed, (name, users - allowed)


def test_oracle_imports_nothing_of_the_cuda_path():
    for path in _py_files(os.path.join(ROOT, "oracle")):
        mods = [m for m, _ in _imports(path)]
        assert not [m for m in mods if m.startswith("decoder_only_transformer_int4_b200")], path
        assert "ctypes" not in mods and "torch" not in mods, (path, mods)


def test_cuda_sources_include_only_their_own_headers():
    csrc = os.path.join(PKG, "csrc")
    inc = re.compile(r'^\s*#\s*include\s*"([^"]+)"', re.M)
    for name in sorted(os.listdir(csrc)):
        for h in inc.findall(open(os.path.join(csrc, name)).read()):
            target = os.path.normpath(os.path.join(csrc, h))
            assert target.startswith(csrc) or target == os.path.join(ROOT, "include", "ms.h"), (name, h)


def test_binding_refuses_to_import_without_its_library(tmp_path):
    pkg = tmp_path / "unbuilt_binding"
    pkg.mkdir()
    shutil.copy(os.path.join(PKG, "__init__.py"), pkg / "__init__.py")
    spec = importlib.util.spec_from_file_location("unbuilt_binding", str(pkg / "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError, match="is missing"):
        spec.loader.exec_module(mod)
