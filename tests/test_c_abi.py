"""The C ABI from C: ``tests/c_abi_check.c`` compiled as strict C11 against
``include/*.h``, linked with the library and run (CPU only; every call it makes
ends in a host-side argument check, none reaches a GPU)."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_caller_compiles_links_and_gets_the_documented_statuses(tmp_path):
    from sub_bit_weight_b200 import build
    lib = build.build()
    exe = tmp_path / "c_abi_check"
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", str(exe),
           "-L", os.path.dirname(lib), "-llittlebit", "-Wl,-rpath," + os.path.dirname(lib)]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "OK", r.stdout + r.stderr
