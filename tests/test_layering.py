"""The oracle stays test infrastructure: the product path neither imports it
nor shares source with it.  CPU only (reads the sources)."""
import ast
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PRODUCT_PY = (glob.glob(os.path.join(ROOT, "int4_routed_expert_renorm_b200", "**", "*.py"), recursive=True)
              + glob.glob(os.path.join(ROOT, "synth", "**", "*.py"), recursive=True))
NATIVE = (glob.glob(os.path.join(ROOT, "int4_routed_expert_renorm_b200", "csrc", "*"))
          + glob.glob(os.path.join(ROOT, "include", "*")) + glob.glob(os.path.join(ROOT, "synth", "csrc", "*")))


def _oracle_imports(tree):
    """(node, enclosing function name or None) for every import of the oracle package."""
    found = []

    def visit(node, fn):
        for child in ast.iter_child_nodes(node):
            name = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else fn
            if isinstance(child, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in child.names):
                found.append((child, fn))
            if isinstance(child, ast.ImportFrom) and (child.module or "").split(".")[0] == "oracle":
                found.append((child, fn))
            visit(child, name)

    visit(tree, None)
    return found


def _parse(path):
    with open(path) as f:
        return ast.parse(f.read(), path)


def test_product_python_never_imports_the_oracle():
    assert PRODUCT_PY
    for p in PRODUCT_PY:
        assert not _oracle_imports(_parse(p)), p


def test_bench_imports_the_oracle_only_in_its_cpu_leg():
    """bench.py imports the oracle only in the functions of its CPU leg:
    oracle_sample and the per-process worker it runs, _oracle_tokens."""
    found = _oracle_imports(_parse(os.path.join(ROOT, "bench.py")))
    assert found and all(fn in ("oracle_sample", "_oracle_tokens") for _, fn in found)
    src = open(os.path.join(ROOT, "bench.py")).read()
    # every use of the worker besides its definition lies inside oracle_sample
    assert src.count("_oracle_tokens") == len(re.findall(r"_oracle_tokens", src[src.index("def oracle_sample"):
                                                                             src.index("def rank_batches")])) + 1


def test_entry_imports_the_oracle_only_to_build_it_and_in_smoke():
    found = _oracle_imports(_parse(os.path.join(ROOT, "__graft_entry__.py")))
    for node, fn in found:
        if fn == "build":
            assert isinstance(node, ast.ImportFrom) and node.module == "oracle.cref"
            assert [a.name for a in node.names] == ["build"]
        else:
            assert fn == "_smoke_case", fn


def test_native_sources_share_nothing_with_the_oracle():
    assert NATIVE
    inc = re.compile(r'^\s*#\s*include\s*[<"]([^>"]+)[>"]', re.M)
    for p in NATIVE:
        with open(p, errors="replace") as f:
            text = f.read()
        for h in inc.findall(text):
            assert "oracle" not in h and "moe_ref" not in h, (p, h)
    with open(os.path.join(ROOT, "oracle", "c", "moe_ref.c")) as f:
        ref = f.read()
    assert inc.findall(ref) and all(h in ("math.h", "stdint.h", "stdlib.h", "string.h") for h in inc.findall(ref))
    assert '#include "' not in ref
