"""The product path and the oracle stay apart: nothing in the package imports the oracle,
the oracle imports nothing of the package, and bench.py reaches the oracle only inside its
CPU-baseline / reference-arm code.  Checked on the sources (CPU only)."""
import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "hybrid_deltanet_attention_kva_b200")


def _imports(path):
    tree = ast.parse(open(path).read())
    out = []
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            out += [(a.name, node) for a in node.names]
        elif isinstance(node, ast.ImportFrom) and node.module:
            out.append((node.module, node))
    return tree, out


def test_package_never_imports_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith(".py"):
                _, imps = _imports(os.path.join(dirpath, f))
                assert not any(m.split(".")[0] == "oracle" for m, _ in imps), f
            if f.endswith((".cu", ".cuh", ".h", ".cpp")):
                assert "kva_ref" not in open(os.path.join(dirpath, f)).read(), f


def test_oracle_imports_nothing_of_the_package():
    _, imps = _imports(os.path.join(ROOT, "oracle", "kva_ref.py"))
    for m, _ in imps:
        assert m.split(".")[0] not in ("hybrid_deltanet_attention_kva_b200", "torch", "bench"), m


def test_bench_imports_the_oracle_only_in_its_cpu_legs():
    tree, _ = _imports(os.path.join(ROOT, "bench.py"))
    allowed = {"OracleSample"}
    for node in tree.body:                       # nothing at module level
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            names = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module]
            assert not any(n and n.split(".")[0] == "oracle" for n in names)
    for node in ast.walk(tree):
        if isinstance(node, (ast.FunctionDef, ast.ClassDef)) and node.name not in allowed:
            for sub in ast.walk(node):
                if isinstance(sub, ast.ImportFrom) and sub.module and sub.module.startswith("oracle"):
                    # an import inside a function that is not part of the CPU legs
                    parents = [n.name for n in ast.walk(tree) if isinstance(n, ast.ClassDef)
                               and sub in list(ast.walk(n))]
                    assert set(parents) & allowed, node.name
