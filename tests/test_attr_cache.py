"""The per-device record of raised shared-memory limits, checked on the host (no GPU).

CUDA keeps a kernel's dynamic shared-memory limit per device; the library
records what it raised per (device, kernel), under a lock, so that a process
driving several GPUs, or several threads, never skips a raise it needs.
"""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_attr_cache_host_logic(tmp_path):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("no host C++ compiler")
    exe = tmp_path / "attr_cache_check"
    src = os.path.join(ROOT, "tests", "attr_cache_check.cpp")
    inc = os.path.join(ROOT, "sub_bit_weight_b200", "csrc")
    subprocess.run([gxx, "-std=c++17", "-O1", "-Wall", "-Werror", "-pthread", "-I", inc, src, "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "attr cache ok" in r.stdout
