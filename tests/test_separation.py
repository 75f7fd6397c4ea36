"""The oracle and the CUDA path share no code.

The library (``latentmoe_fwd_b200/``, ``include/``) never imports, links or
names the oracle; the oracle never loads the library; the seeded input
generator imports neither. ``bench.py`` reaches the oracle only from its CPU
baseline and reference-arm functions. Static checks on the sources (CPU).
"""
import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _files(sub, exts):
    for dirpath, _, names in os.walk(os.path.join(ROOT, sub)):
        if "_build" in dirpath or "__pycache__" in dirpath:
            continue
        for n in names:
            if n.endswith(exts):
                yield os.path.join(dirpath, n)


def _imports(path):
    tree = ast.parse(open(path).read(), path)
    out = []
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            out += [a.name for a in node.names]
        elif isinstance(node, ast.ImportFrom):
            out.append(("." * node.level) + (node.module or ""))
    return out


def test_library_sources_never_name_the_oracle():
    hits = []
    for path in _files("latentmoe_fwd_b200", (".py", ".cu", ".cuh", ".h", ".cpp")):
        if re.search(r"\boracle\b", open(path, errors="replace").read()):
            hits.append(os.path.relpath(path, ROOT))
    for path in _files("include", (".h",)):
        if re.search(r"\boracle\b", open(path).read()):
            hits.append(os.path.relpath(path, ROOT))
    assert not hits, hits


def test_oracle_never_loads_the_library():
    for path in _files("oracle", (".py",)):
        mods = _imports(path)
        assert not any(m.split(".")[0] in ("latentmoe_fwd_b200", "ctypes", "torch") for m in mods), (path, mods)
        assert "liblmoe" not in open(path).read(), path


def test_input_generator_imports_neither_side():
    for path in _files("lmoe_inputs", (".py",)):
        mods = [m.split(".")[0] for m in _imports(path)]
        assert "oracle" not in mods and "latentmoe_fwd_b200" not in mods, (path, mods)


def test_bench_reaches_the_oracle_only_from_its_cpu_legs():
    path = os.path.join(ROOT, "bench.py")
    tree = ast.parse(open(path).read(), path)
    allowed = {"oracle_tokens_per_s"}
    for node in tree.body:          # no module-level import of the oracle
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            names = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module or ""]
            assert not any(n.split(".")[0] == "oracle" for n in names)
    for fn in ast.walk(tree):
        if not isinstance(fn, ast.FunctionDef):
            continue
        for node in ast.walk(fn):
            if isinstance(node, ast.ImportFrom) and (node.module or "").split(".")[0] == "oracle":
                assert fn.name in allowed, fn.name
            if isinstance(node, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in node.names):
                assert fn.name in allowed, fn.name
