"""Build the CUDA library ``libnvq.so`` in-tree for sm_100a (B200).

``build(debug=True)`` builds ``libnvq_debug.so`` from the same sources with
NVQ_DEBUG defined: every kernel then checks its computed global accesses
against the extents of the buffers it was given and reports a failed check in
the device status word (NVQ_STATUS_BOUNDS) instead of making the access.  The
package loads it in place of ``libnvq.so`` when NVQ_DEBUG=1 is set.

One translation unit (``csrc/nvq.cu``) holds the C ABI and includes the
kernels; the CUDA runtime is linked statically and the driver API is reached
through ``cudaGetDriverEntryPoint``, so the library loads on a machine
without a GPU driver (it then reports errors from its entry points).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libnvq.so")
LIB_DEBUG = os.path.join(HERE, "libnvq_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-cudart", "static",
    # scale arithmetic must stay IEEE FP32 round-to-nearest in program order
    "-fmad=false", "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cu", ".cuh"))]


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    deps = sources() + [os.path.join(ROOT, "include", "nvq.h"), __file__]
    if not force and os.path.exists(lib) and all(os.path.getmtime(lib) >= os.path.getmtime(d) for d in deps):
        return lib
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = [NVCC, *NVCC_FLAGS, *(["-DNVQ_DEBUG"] if debug else []), *(["-Xptxas", "-v"] if verbose else []),
           os.path.join(CSRC, "nvq.cu"), "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
