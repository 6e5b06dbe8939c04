"""The oracle and the CUDA path share no code, checked on the sources:

* no module of the package imports the oracle (the product path has no CPU
  fallback to reach it through);
* the oracle imports nothing from the package;
* no CUDA or C source of the package, and no public header, includes a file
  from the oracle;
* the only module the two sides have in common is the seeded input generator,
  which holds none of the method's arithmetic: it imports no part of either.
"""
import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "newton_schulz_09_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _py_files(folder):
    for dirpath, _, files in os.walk(folder):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(dirpath, f)


def _imports(path):
    tree = ast.parse(open(path, encoding="utf-8").read(), filename=path)
    out = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            out.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            if node.level == 0 and node.module:
                out.add(node.module.split(".")[0])
            elif node.level > 0:
                out.add("." + (node.module or ""))
    return out


def test_package_never_imports_the_oracle():
    for path in _py_files(PKG):
        assert "oracle" not in _imports(path), path


def test_oracle_never_imports_the_package():
    for path in _py_files(ORACLE):
        assert "newton_schulz_09_b200" not in _imports(path), path


def test_native_sources_include_nothing_from_the_oracle():
    inc = re.compile(r'^\s*#\s*include\s*[<"]([^>"]+)[>"]', re.M)
    native = [os.path.join(PKG, "csrc", f) for f in os.listdir(os.path.join(PKG, "csrc"))]
    native += [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))]
    for path in native:
        for name in inc.findall(open(path, encoding="utf-8").read()):
            assert "oracle" not in name, (path, name)


def test_input_generator_imports_neither_side():
    deps = _imports(os.path.join(PKG, "synthetic.py"))
    assert "oracle" not in deps
    assert not any(d.startswith(".") and d != "." for d in deps), deps
    assert "." not in deps, deps
