"""GPU parity of the block-scaled GEMM (tcgen05) against the oracle's FP64
sum over the oracle-dequantized operands.  Acceptance: for every checked row
max_n |D - Y| / ||Y[row, :]||_2 <= 2e-3.  Small shapes compare every output;
the full-size workloads compare sampled rows (first and last row of 128-row
tiles plus random rows) in the same launch configuration the benchmark uses."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import act, bits, check_gemm, sample_rows, wgt

pytestmark = pytest.mark.gpu

nvq = pytest.importorskip("microscaling_quantized_linear_b200")


ELEM = {"mxfp8": "e4m3", "mxfp8_e5m2": "e5m2"}


def gpu_linear(fmt, x, w, bias=None, ldo=None, guard_rows=0):
    M, K = x.shape
    N = w.shape[0]
    xd, wd = x.cuda(), w.cuda()
    wc, ws, wg = nvq.quantize_weight(fmt, wd)
    if fmt == "nvfp4":
        ac, as_, ag = nvq.nvfp4_quantize(xd)
    else:
        ac, as_ = nvq.mxfp8_quantize(xd, elem=ELEM[fmt])
        ag = None
    # NaN-filled output (and padding columns, and guard rows past M): any tile
    # the kernel fails to write, or any element it writes by mistake, shows up
    out = torch.full((M + guard_rows, ldo or N), float("nan"), dtype=torch.bfloat16, device="cuda")[:M, :N]
    bd = bias.cuda() if bias is not None else None
    D = nvq.block_scaled_linear(fmt, ac, as_, ag, wc, ws, wg, M, N, K, bias=bd, out=out)
    assert nvq.device_status() == 0
    return D


def oracle_linear(fmt, x, w, rows=None, bias=None):
    M, K = x.shape
    N = w.shape[0]
    if fmt == "nvfp4":
        ac, as_, ag = oracle.nvfp4_quantize(bits(x))
        wc, ws, wg = oracle.nvfp4_quantize(bits(w))
        A = oracle.nvfp4_dequantize(ac, as_, ag, M, K)
        B = oracle.nvfp4_dequantize(wc, ws, wg, N, K)
    else:
        e = ELEM[fmt]
        ac, as_ = oracle.mxfp8_quantize(bits(x), elem=e)
        wc, ws = oracle.mxfp8_quantize(bits(w), elem=e)
        A = oracle.mxfp8_dequantize(ac, as_, M, K, elem=e)
        B = oracle.mxfp8_dequantize(wc, ws, N, K, elem=e)
    return oracle.gemm_rows(A, B, rows, bias_bits=None if bias is None else bits(bias.reshape(1, -1)))


SMALL = [
    # fmt, M, N, K.  M % 256 == 0 and N % 256 == 0 run on CTA pairs (256 x 256
    # tiles); otherwise one CTA per tile, 256 wide if N allows, else 192 or 128.
    ("nvfp4", 128, 128, 256),
    ("nvfp4", 256, 384, 512),
    ("nvfp4", 384, 512, 768),
    ("nvfp4", 1024, 768, 512),
    ("mxfp8", 128, 128, 128),
    ("mxfp8", 256, 384, 384),
    ("mxfp8", 384, 512, 640),
    ("mxfp8", 512, 512, 384),          # CTA-pair kernel
    ("mxfp8", 256, 256, 128),          # CTA-pair kernel, one K stage
    ("mxfp8_e5m2", 128, 128, 128),     # E5M2 x E5M2, one CTA
    ("mxfp8_e5m2", 512, 512, 384),     # E5M2, CTA pairs
    ("mxfp8_e5m2", 256, 384, 256),     # E5M2, 256 x 192 pair tiles (two accumulators)
]


def test_tiny_workload_full_output():
    x, w = act("tiny"), workloads.weight("tiny")
    D = gpu_linear("nvfp4", x, w).float().cpu().numpy()
    Y = oracle_linear("nvfp4", x, w)
    check_gemm(D, Y)


@pytest.mark.parametrize("fmt,M,N,K", SMALL)
def test_small_shapes_full_output(fmt, M, N, K):
    x = workloads.normal(M, K, seed=40 + M)
    w = workloads.normal(N, K, seed=41 + N, std=0.05)
    D = gpu_linear(fmt, x, w).float().cpu().numpy()
    check_gemm(D, oracle_linear(fmt, x, w))


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp8"])
def test_bias_and_output_pitch(fmt):
    M, N, K = 256, 512, 512
    x = workloads.normal(M, K, seed=50)
    w = workloads.normal(N, K, seed=51, std=0.05)
    b = workloads.bias(N)
    D = gpu_linear(fmt, x, w, bias=b, ldo=N + 64)
    full = D.as_strided((M, N + 64), (N + 64, 1))
    assert torch.isnan(full[:, N:]).all(), "padding columns of the output were written"
    check_gemm(D.float().cpu().numpy(), oracle_linear(fmt, x, w, bias=b))


RAGGED = [
    # row counts that are not multiples of 128 (N a multiple of 8): tensor-map
    # loads read zeros past the end, stores are clipped, bias is read only for n < N
    ("nvfp4", 1, 256, 256),
    ("nvfp4", 100, 200, 256),
    ("nvfp4", 300, 520, 512),          # CTA pairs, last pair tile mostly empty
    ("mxfp8", 129, 136, 384),
    ("mxfp8", 1000, 1000, 256),
    ("mxfp8_e5m2", 700, 336, 256),
]


@pytest.mark.parametrize("fmt,M,N,K", RAGGED)
def test_ragged_shapes_with_bias(fmt, M, N, K):
    x = workloads.normal(M, K, seed=70 + M % 97)
    w = workloads.normal(N, K, seed=71 + N % 89, std=0.05)
    b = workloads.bias(N)
    ldo = (N + 7) // 8 * 8 + 8
    D = gpu_linear(fmt, x, w, bias=b, ldo=ldo, guard_rows=3)
    full = D.as_strided((M + 3, ldo), (ldo, 1))
    assert torch.isnan(full[:M, N:]).all(), "columns past N were written"
    assert torch.isnan(full[M:]).all(), "rows past M were written"
    check_gemm(D.float().cpu().numpy(), oracle_linear(fmt, x, w, bias=b))


MANY_TILES = [
    # several output tiles per persistent CTA: both tensor-memory accumulators,
    # barrier phase wrap-around, and (BN = 192) tiles that start mid scale tile
    ("nvfp4", 128 * 48, 384 * 4, 256),     # BN 192, 384 tiles
    ("nvfp4", 128 * 40, 256 * 3, 512),     # BN 256 (one accumulator), 240 tiles
    ("mxfp8", 128 * 40, 640, 256),         # BN 128, 200 tiles
    ("mxfp8", 128 * 36, 384 * 3, 384),     # BN 192, 216 tiles
]


@pytest.mark.parametrize("fmt,M,N,K", MANY_TILES)
def test_many_tiles_per_cta(fmt, M, N, K):
    x = workloads.normal(M, K, seed=60 + M % 97)
    w = workloads.normal(N, K, seed=61 + N % 89, std=0.05)
    rows = sample_rows(M)
    D = gpu_linear(fmt, x, w)
    Dr = D[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    check_gemm(Dr, oracle_linear(fmt, x, w, rows=rows))
    assert torch.isfinite(D).all(), "some output tile was not written"


def test_zero_activation_gives_zero_output():
    x = torch.zeros(128, 256, dtype=torch.bfloat16)
    w = workloads.weight("tiny")
    D = gpu_linear("nvfp4", x, w)
    assert (D == 0).all()


def test_gemm_deterministic():
    x, w = act("tiny"), workloads.weight("tiny")
    a = gpu_linear("nvfp4", x, w)
    b = gpu_linear("nvfp4", x, w)
    assert torch.equal(a, b)


FULL = [
    ("ffup", "nvfp4", 1),
    ("ffdown", "mxfp8", 1),
    ("qkv4", "nvfp4", 8),
]


@pytest.mark.parametrize("name,fmt,every", FULL, ids=[f[0] for f in FULL])
def test_full_size_workloads_sampled_rows(name, fmt, every):
    x, w = act(name), wgt(name)
    rows = sample_rows(x.shape[0], per_tile_every=every)
    D = gpu_linear(fmt, x, w)
    Dr = D[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    Y = oracle_linear(fmt, x, w, rows=rows)
    check_gemm(Dr, Y)


SINGLE_CTA_SCRIPT = r"""
import sys, numpy as np, torch
sys.path.insert(0, ROOT_DIR)
sys.path.insert(0, TEST_DIR)
import test_gpu_gemm as t
from gpu_common import check_gemm, sample_rows
import workloads
for fmt, M, N, K in [("nvfp4", 1024, 768, 512), ("mxfp8", 512, 512, 384), ("nvfp4", 4608, 12288, 3072),
                     ("nvfp4", 300, 520, 512), ("mxfp8_e5m2", 700, 336, 256)]:
    x = workloads.normal(M, K, seed=90 + M % 13)
    w = workloads.normal(N, K, seed=91 + N % 11, std=0.05)
    rows = sample_rows(M, per_tile_every=4)
    D = t.gpu_linear(fmt, x, w)
    Dr = D[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    err = check_gemm(Dr, t.oracle_linear(fmt, x, w, rows=rows))
    print(fmt, M, N, K, "max row err %.2e" % err)
print("OK")
"""


def test_single_cta_kernel_on_pair_shapes():
    # The library picks CTA pairs for these shapes; NVQ_GEMM_PAIRS=0 (read
    # when the library loads, hence a fresh process) forces the one-CTA
    # kernel, which must give the same answers.
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    root = os.path.dirname(here)
    env = dict(os.environ, NVQ_GEMM_PAIRS="0")
    script = SINGLE_CTA_SCRIPT.replace("ROOT_DIR", repr(root)).replace("TEST_DIR", repr(here))
    out = subprocess.run([sys.executable, "-c", script], env=env,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0 and out.stdout.strip().endswith("OK"), out.stdout + out.stderr
