"""The CUDA path and the oracle stay apart, and the product has no fallback (CPU).

* Nothing in the package (``sub_bit_weight_b200``: binding, builder, input
  generators, CUDA sources) imports, includes or opens anything under
  ``oracle/``; the oracle imports nothing of the package (the seeded input
  generators, which hold none of the layer arithmetic, are handed to it by the
  tests).
* Importing the binding where the compiled library is absent raises
  ImportError at once: no call can silently take another route.
"""

import ast
import os
import re
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sub_bit_weight_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _py_imports(path):
    tree = ast.parse(open(path).read(), filename=path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            if node.level:                      # relative: stays inside its own package
                continue
            names.add(node.module or "")
    return names


def _files(top, exts):
    for d, _, fs in os.walk(top):
        if "__pycache__" in d:
            continue
        for f in fs:
            if f.endswith(exts):
                yield os.path.join(d, f)


def test_package_never_reaches_the_oracle():
    for f in _files(PKG, (".py",)):
        bad = [n for n in _py_imports(f) if n == "oracle" or n.startswith("oracle.")]
        assert not bad, (f, bad)
        assert "littlebit_oracle" not in open(f).read(), f
    for f in _files(PKG, (".cu", ".cuh", ".h")):
        text = open(f).read()
        assert "oracle" not in text.lower(), f
    for f in _files(os.path.join(ROOT, "include"), (".h",)):
        assert "oracle" not in open(f).read().lower(), f


def test_oracle_never_reaches_the_package():
    for f in _files(ORACLE, (".py",)):
        bad = [n for n in _py_imports(f) if n.startswith("sub_bit_weight_b200")]
        assert not bad, (f, bad)
    for f in _files(ORACLE, (".c", ".h")):
        includes = re.findall(r'#include\s*[<"]([^>"]+)[>"]', open(f).read())
        assert all(i in ("math.h", "stdint.h", "stdlib.h", "string.h", "stddef.h", "stdio.h") for i in includes), \
            (f, includes)


def test_binding_refuses_to_load_without_the_library(tmp_path):
    # a copy of the package without its compiled library
    dst = tmp_path / "sub_bit_weight_b200"
    shutil.copytree(PKG, dst, ignore=shutil.ignore_patterns("*.so", "__pycache__", "csrc"))
    assert not any(p.suffix == ".so" for p in dst.iterdir())
    code = ("import sys; sys.path.insert(0, sys.argv[1])\n"
            "try:\n"
            "    import sub_bit_weight_b200.lib\n"
            "except ImportError as e:\n"
            "    print('IMPORT_ERROR', e); sys.exit(0)\n"
            "print('LOADED'); sys.exit(1)\n")
    r = subprocess.run([sys.executable, "-c", code, str(tmp_path)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "IMPORT_ERROR" in r.stdout and "liblittlebit.so" in r.stdout
