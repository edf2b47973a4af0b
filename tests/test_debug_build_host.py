"""The debug build of the C-ABI library (NVQ_DEBUG), checked without a GPU.

libnvq_debug.so is compiled from the same sources with NVQ_DEBUG defined, so
that every kernel checks its computed global accesses against the extents of
the buffers it was given and reports a failed check as NVQ_STATUS_BOUNDS.
Here: it builds, it exports exactly the entry points of the normal build,
nvq_debug_build tells the two apart, and the package loads the debug build
when NVQ_DEBUG=1 is set at import.
"""
import ctypes
import importlib.util
import os
import subprocess
import sys

import microscaling_quantized_linear_b200 as nvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def build_debug():
    spec = importlib.util.spec_from_file_location(
        "_nvq_build_for_test", os.path.join(ROOT, "microscaling_quantized_linear_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build(debug=True)


def exported(path):
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    return {line.split()[-1] for line in out.splitlines() if " T " in line}


def test_debug_build_exports_the_same_entry_points():
    lib = build_debug()
    assert exported(lib) == exported(nvq.LIB_PATH)
    assert set(nvq.EXPORTED) <= exported(lib)


def test_debug_build_reports_itself():
    lib = build_debug()
    assert ctypes.CDLL(lib).nvq_debug_build() == 1
    assert nvq._lib.nvq_debug_build() == 0 and not nvq.DEBUG_BUILD
    assert nvq.NVQ_STATUS_BOUNDS == 8


def test_package_loads_the_debug_build_on_request():
    build_debug()
    script = ("import microscaling_quantized_linear_b200 as nvq; "
              "print(nvq.DEBUG_BUILD, nvq.LIB_PATH.endswith('libnvq_debug.so'))")
    out = subprocess.run([sys.executable, "-c", script], env=dict(os.environ, NVQ_DEBUG="1"), cwd=ROOT,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.split() == ["True", "True"]
