"""The product path and the oracle stay independent: the package (binding, layer,
kernels) never imports or reads anything under oracle/, the oracle imports nothing from
the package but the seeded input generators, and no CUDA source names the oracle.
CPU only."""
import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "routing_dispatch_expert_moe_b200")


def _imports(path):
    tree = ast.parse(open(path, encoding="utf-8").read())
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            mod = node.module or ""
            names.add(mod)
            names.update(f"{mod}.{a.name}" if mod else a.name for a in node.names)
    return names


def test_package_never_imports_the_oracle():
    for f in os.listdir(PKG):
        if f.endswith(".py"):
            bad = [n for n in _imports(os.path.join(PKG, f)) if n == "oracle" or n.startswith("oracle.")]
            assert not bad, (f, bad)
    for f in os.listdir(os.path.join(PKG, "csrc")):
        src = open(os.path.join(PKG, "csrc", f), encoding="utf-8").read()
        assert "oracle" not in src.lower(), f


def test_oracle_imports_only_the_input_generators():
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith(".py"):
            for n in _imports(os.path.join(ROOT, "oracle", f)):
                if n.startswith("routing_dispatch_expert_moe_b200"):
                    assert n in ("routing_dispatch_expert_moe_b200", "routing_dispatch_expert_moe_b200.inputs"), (f, n)
