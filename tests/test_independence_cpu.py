"""The oracle and the CUDA path share no code: the product package never imports the oracle or the input
generator, the oracle never imports the product, and the input generator holds no step arithmetic of
either side (it imports neither).  Checked on the sources' import statements."""
import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _imports(path):
    tree = ast.parse(open(path).read(), filename=path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.level == 0 and node.module:
            names.add(node.module.split(".")[0])
    return names


def _py_files(pkg):
    d = os.path.join(ROOT, pkg)
    return [os.path.join(dp, f) for dp, _, fs in os.walk(d) for f in fs if f.endswith(".py")]


def test_product_package_imports_neither_oracle_nor_generator():
    for p in _py_files("decodability_aware_token_b200"):
        bad = _imports(p) & {"oracle", "focus_synth", "tests", "bench"}
        assert not bad, f"{p} imports {bad}"


def test_oracle_imports_no_product_code():
    for p in _py_files("oracle"):
        bad = _imports(p) & {"decodability_aware_token_b200", "focus_synth", "tests", "bench"}
        assert not bad, f"{p} imports {bad}"


def test_generator_imports_neither_side():
    for p in _py_files("focus_synth"):
        bad = _imports(p) & {"decodability_aware_token_b200", "oracle", "tests", "bench"}
        assert not bad, f"{p} imports {bad}"


def test_cuda_sources_reference_no_oracle():
    csrc = os.path.join(ROOT, "decodability_aware_token_b200", "csrc")
    for f in os.listdir(csrc):
        if f.endswith((".cu", ".cuh", ".h")):
            assert "oracle" not in open(os.path.join(csrc, f)).read().lower(), f
