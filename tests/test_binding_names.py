"""Static check of the Python binding and the benchmark: every name they
read is bound somewhere in the same file (a definition, an import, an
assignment or a parameter) or is a builtin.  Much of the binding only runs
with a GPU, so a name lost in an edit would otherwise surface there first."""
import ast
import builtins
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FILES = ["nvfp4_quantization_amax_b200/_abi.py", "nvfp4_quantization_amax_b200/__init__.py",
         "nvfp4_quantization_amax_b200/build.py", "bench.py", "__graft_entry__.py"]


def unbound_names(path):
    with open(path) as f:
        tree = ast.parse(f.read(), path)
    bound = set(dir(builtins)) | {"__file__", "__name__"}
    for node in ast.walk(tree):
        if isinstance(node, (ast.FunctionDef, ast.AsyncFunctionDef, ast.ClassDef)):
            bound.add(node.name)
        elif isinstance(node, ast.Import):
            bound.update((a.asname or a.name).split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            bound.update(a.asname or a.name for a in node.names)
        elif isinstance(node, ast.Name) and not isinstance(node.ctx, ast.Load):
            bound.add(node.id)
        elif isinstance(node, ast.arg):
            bound.add(node.arg)
        elif isinstance(node, ast.ExceptHandler) and node.name:
            bound.add(node.name)
    used = {n.id for n in ast.walk(tree) if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Load)}
    return sorted(used - bound)


@pytest.mark.parametrize("rel", FILES)
def test_every_name_read_is_bound(rel):
    assert unbound_names(os.path.join(ROOT, rel)) == []
