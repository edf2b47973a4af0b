"""The boundary is a C ABI: a plain C99 program that includes include/nvq.h
and links the built library compiles without warnings and runs its
host-only calls (size helpers, status strings, the wait-limit hook, host
argument checks) on a machine without a GPU (tests/c_abi_check.c)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "microscaling_quantized_linear_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_caller_builds_and_runs(tmp_path):
    lib = os.path.join(PKG, "libnvq.so")
    assert os.path.exists(lib), "build it with __graft_entry__.build()"
    exe = str(tmp_path / "c_abi_check")
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                         "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_check.c"),
                         "-o", exe, "-L", PKG, "-l:libnvq.so", "-Wl,-rpath," + PKG],
                        capture_output=True, text=True, timeout=120)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "C ABI OK" in run.stdout
