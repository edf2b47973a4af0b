"""The debug build (NVQ_DEBUG) on the GPU: every kernel of the path runs with
its bounds checks on, reports none, and gives the same results.

In libnvq_debug.so every kernel checks each global access whose address it
computes against the extent of the buffer it was given; a failed check sets
NVQ_STATUS_BOUNDS and skips the access (nothing traps).  The script below
runs in a child process with NVQ_DEBUG=1, so the package loads the debug
build.  It first drives the report path with nvq_probe_bounds (one failing
check, no memory access), then runs every quantizer and GEMM kernel once on
shapes with ragged and pitched edges: each call must leave the status word
clean, quantizer outputs must equal the oracle's bit for bit, GEMM outputs
must meet the tolerance, and the fused epilogue on exact-grid operands must
equal the oracle's codes and scales bit for bit.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import os, sys
sys.path[:0] = [os.path.join(ROOT, "tests"), ROOT]
import numpy as np
import torch
import microscaling_quantized_linear_b200 as nvq
assert nvq.DEBUG_BUILD, nvq.LIB_PATH
import oracle
import workloads
from gpu_common import bits, check_gemm
from test_gpu_gemm import gpu_linear, oracle_linear
from test_gpu_fused import quantize_both, gpu_fused

torch.cuda.set_device(0)
assert nvq.device_status() == 0
nvq.probe_bounds()
assert nvq.device_status() == nvq.NVQ_STATUS_BOUNDS
assert nvq.device_status() == 0


def clean(what):
    st = nvq.device_status()
    assert st == 0, (what, st)


def nvfp4_case(name, x, calib=None, noalloc=False):
    M, K = x.shape
    xd = x.cuda()
    if noalloc:
        c = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
        s = torch.empty(nvq.scale_bytes("nvfp4", M, K), dtype=torch.uint8, device="cuda")
        g = torch.empty(1, dtype=torch.float32, device="cuda")
        nvq.nvfp4_quantize_noalloc(xd, c, s, g)
    else:
        amax = None if calib is None else torch.tensor([calib], dtype=torch.float32, device="cuda")
        c, s, g = nvq.nvfp4_quantize(xd, calib_amax=amax)
    clean(name)
    oc, osf, og = oracle.nvfp4_quantize(bits(x), calib_amax=calib)
    assert np.array_equal(c.cpu().numpy(), oc), name
    assert np.array_equal(s.cpu().numpy(), osf), name
    assert np.float32(g.item()).tobytes() == np.float32(og).tobytes(), name


def pitched(M, K, pad, seed):
    return workloads.normal(M, K + pad, seed=seed)[:, :K]


nvfp4_case("one-pass", workloads.activation("ffup", seed=3))
nvfp4_case("cluster", workloads.normal(100, 256, seed=4))
nvfp4_case("two-pass", workloads.normal(2048, 16384, seed=5))
nvfp4_case("two-pass pitched", pitched(1500, 12288, 64, 6))
nvfp4_case("calibrated", workloads.normal(300, 1024, seed=7), calib=6.0)
nvfp4_case("no-alloc", workloads.normal(1000, 2048, seed=8), noalloc=True)
nvfp4_case("one-pass pitched", pitched(777, 3072, 32, 9))

for elem in ("e4m3", "e5m2"):
    for rule in ("floor", "ceil"):
        for x in (workloads.normal(500, 1024, seed=10), pitched(130, 2048, 96, 11)):
            c, s = nvq.mxfp8_quantize(x.cuda(), elem=elem, rule=rule)
            clean("mxfp8 %s %s" % (elem, rule))
            oc, osf = oracle.mxfp8_quantize(bits(x), elem=elem, rule=rule)
            assert np.array_equal(c.cpu().numpy(), oc) and np.array_equal(s.cpu().numpy(), osf), (elem, rule)

GEMMS = [
    ("nvfp4", 100, 384, 256, True),       # one CTA, 128-wide tiles
    ("nvfp4", 128, 37888, 256, False),    # one CTA, 256-wide tiles
    ("nvfp4", 512, 768, 512, True),       # CTA pairs
    ("nvfp4", 300, 520, 512, False),      # CTA pairs, ragged M and N
    ("nvfp4", 1, 12288, 3072, False),     # split-K clusters
    ("nvfp4", 29, 256, 4096, True),       # split-K, 8 CTAs per cluster, ragged N
    ("mxfp8", 24, 3072, 12288, True),     # split-K, MXFP8
    ("mxfp8", 512, 1024, 512, False),     # CTA pairs, MXFP8
]
for fmt, M, N, K, use_bias in GEMMS:
    x = workloads.normal(M, K, seed=M + 1)
    w = workloads.normal(N, K, seed=N + 2, std=0.05)
    b = workloads.bias(N) if use_bias else None
    D = gpu_linear(fmt, x, w, bias=b)              # asserts a clean status word
    check_gemm(D.float().cpu().numpy(), oracle_linear(fmt, x, w, bias=b))

for M, N, K in ((1, 12288, 3072), (7, 1000, 2048), (16, 9216, 3072)):   # one-launch short-batch linear
    x = workloads.normal(M, K, seed=M + 9)
    w = workloads.normal(N, K, seed=N + 3, std=0.05)
    wc, ws, wg = nvq.quantize_weight("nvfp4", w.cuda())
    ac = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    asf = torch.empty(nvq.scale_bytes("nvfp4", M, K), dtype=torch.uint8, device="cuda")
    D = nvq.nvfp4_linear_short_m(x.cuda(), wc, ws, wg, N, a_codes=ac, a_scales=asf)
    clean("short-M linear %d x %d x %d" % (M, N, K))
    oc, osf, _ = oracle.nvfp4_quantize(bits(x))
    assert np.array_equal(ac.cpu().numpy(), oc) and np.array_equal(asf.cpu().numpy(), osf)
    check_gemm(D.float().cpu().numpy(), oracle_linear("nvfp4", x, w))

for fmt, M, N, K in (("nvfp4", 384, 768, 512), ("nvfp4", 100, 384, 256), ("mxfp8", 96, 256, 256)):
    if fmt == "nvfp4":
        x, _ = workloads.exact_operand(M, K, seed=M + K, top_row=M // 2)
        w, _ = workloads.exact_operand(N, K, seed=N + 7, top_row=0)
    else:
        x, _ = workloads.exact_operand(M, K, seed=M + K, significands=(1.0, 1.5))
        w, _ = workloads.exact_operand(N, K, seed=N + 7, significands=(1.0, 1.5))
    ops, A, B = quantize_both(fmt, x, w)
    yc, ys = gpu_fused(fmt, ops, M, N, K)          # asserts a clean status word
    oc, osf, _, _, _ = oracle.linear_gelu_mxfp8(A, B)
    assert np.array_equal(yc, oc) and np.array_equal(ys, osf), (fmt, M, N, K)

clean("end")
print("DEBUG BUILD OK")
"""


def test_debug_build_runs_every_kernel_clean():
    lib = os.path.join(ROOT, "microscaling_quantized_linear_b200", "libnvq_debug.so")
    assert os.path.exists(lib), "build it with __graft_entry__.build()"
    env = dict(os.environ, NVQ_DEBUG="1")
    out = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + SCRIPT], env=env, cwd=ROOT,
                         capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stdout[-3000:] + out.stderr[-6000:]
    assert "DEBUG BUILD OK" in out.stdout
