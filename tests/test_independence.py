"""The oracle and the CUDA path share no code and neither imports the other."""
import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = "cross_layer_kv_shared_b200"


def _imports(path):
    with open(path) as f:
        tree = ast.parse(f.read())
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            names.add(node.module.split(".")[0])
    return names


def _py_files(d):
    for root, _, files in os.walk(os.path.join(ROOT, d)):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(root, f)


def test_oracle_imports_neither_the_package_nor_the_generator():
    for p in _py_files("oracle"):
        bad = _imports(p) & {PKG, "synth", "ctypes", "torch"}
        assert not bad, (p, bad)


def test_package_never_imports_the_oracle():
    for p in _py_files(PKG):
        assert "oracle" not in _imports(p), p


def test_generator_holds_no_method_code():
    for p in _py_files("synth"):
        assert not (_imports(p) & {PKG, "oracle"}), p


def test_native_sources_share_nothing_with_the_oracle():
    csrc = os.path.join(ROOT, PKG, "csrc")
    for root, _, files in os.walk(csrc):
        for f in files:
            with open(os.path.join(root, f), errors="ignore") as fh:
                assert "oracle" not in fh.read().lower(), f
