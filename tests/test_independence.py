"""The oracle and the CUDA path are independent: the library package never
imports or loads the oracle (no CPU fallback on the product path), the
oracle never imports the library, and the only module both take from is the
seeded workload generator, which holds none of the method's arithmetic."""
import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _py_files(sub):
    d = os.path.join(ROOT, sub)
    for dirpath, _, files in os.walk(d):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(dirpath, f)


def _imports(path):
    tree = ast.parse(open(path).read(), filename=path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            names.add(node.module.split(".")[0])
    return names


def test_library_does_not_use_the_oracle():
    for path in _py_files("input_adaptive_block_b200"):
        assert "oracle" not in _imports(path), path
        assert "spade_oracle" not in open(path).read(), path
    for dirpath, _, files in os.walk(os.path.join(ROOT, "input_adaptive_block_b200", "csrc")):
        for f in files:
            text = open(os.path.join(dirpath, f)).read()
            assert not re.search(r"\boracle\b", text, re.I), f


def test_oracle_does_not_use_the_library():
    for path in _py_files("oracle"):
        imps = _imports(path)
        assert "input_adaptive_block_b200" not in imps, path
        assert "ctypes" not in imps and "torch" not in imps, path
        assert "libspade" not in open(path).read(), path


def test_shared_workload_module_holds_no_method_arithmetic():
    """spade_workloads may only generate shapes and seeded numbers: it imports
    neither side, and names none of the method's steps."""
    for path in _py_files("spade_workloads"):
        imps = _imports(path)
        assert not {"oracle", "input_adaptive_block_b200"} & imps, path
        text = open(path).read()
        for word in ("softmax", "summarize", "estimate", "select_row", "attention("):
            assert word not in text, (path, word)
