"""Static checks of the product/test boundary: the library and its binding never reach the
oracle, the oracle never reaches the library, and the shared input generator holds no step
of the layer."""
import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "moe_expert_layer_prefix_b200")


def _files(top, exts):
    for d, _, names in os.walk(top):
        for n in names:
            if n.endswith(exts):
                yield os.path.join(d, n)


def _imports(path):
    tree = ast.parse(open(path).read())
    out = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            out |= {a.name.split(".")[0] for a in node.names}
        elif isinstance(node, ast.ImportFrom) and node.module:
            out.add(node.module.split(".")[0])
    return out


def test_product_never_imports_the_oracle_or_the_tests():
    for f in _files(PKG, (".py",)):
        assert not _imports(f) & {"oracle", "tests", "synth"}, f
    for f in _files(PKG, (".cu", ".cuh", ".h")):
        assert "oracle" not in open(f).read(), f


def test_oracle_never_imports_the_library():
    for f in _files(os.path.join(ROOT, "oracle"), (".py",)):
        assert not _imports(f) & {"moe_expert_layer_prefix_b200", "synth", "tests"}, f


def test_input_generator_holds_no_layer_step():
    # synth draws seeded inputs and quantises them into the storage formats; it must not
    # route, dispatch, run an expert or combine (those live in the oracle and the library)
    f = os.path.join(ROOT, "synth", "__init__.py")
    assert not _imports(f) & {"oracle", "moe_expert_layer_prefix_b200", "tests"}
    names = {n.name for n in ast.walk(ast.parse(open(f).read()))
             if isinstance(n, ast.FunctionDef)}
    for step in ("route", "dispatch", "combine", "forward", "expert_ffn", "swiglu"):
        assert not any(step in n for n in names), step


def test_graft_entry_reaches_the_oracle_only_from_smoke():
    tree = ast.parse(open(os.path.join(ROOT, "__graft_entry__.py")).read())
    for fn in (n for n in tree.body if isinstance(n, ast.FunctionDef)):
        mods = set()
        for node in ast.walk(fn):
            if isinstance(node, ast.Import):
                mods |= {a.name.split(".")[0] for a in node.names}
            elif isinstance(node, ast.ImportFrom) and node.module:
                mods.add(node.module.split(".")[0])
        if fn.name != "smoke":
            assert "oracle" not in mods, fn.name
    top = {a.name for n in tree.body if isinstance(n, ast.Import) for a in n.names}
    assert "oracle" not in top
