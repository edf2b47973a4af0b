"""GPU parity of the short-M GEMM path: at M <= 32 block_scaled_linear may
split the K range of each output tile over a cluster of CTAs, each summing
its share into its own FP32 accumulator.  Each CTA then pushes its partial of
every share of the tile into the shared memory of the CTA that finishes that
share, which adds the partials in rank order.

  * the library's plan (nvq_gemm_plan) splits the short-M shapes below and
    leaves the others alone;
  * every output of those shapes meets the GEMM tolerance against the
    oracle's binary64 sum, with bias, an output pitch, ragged N, and NaN
    canaries past N and past M that must survive;
  * on the exact binary grid (workloads.exact_operand) every partial sum is a
    binary32 number whatever the split, so D equals bf16 of the oracle's sum
    bit for bit;
  * NVQ_GEMM_SPLITK=0 (read when the library loads) turns the split off.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import bits, check_gemm
from test_gpu_gemm import gpu_linear, oracle_linear

pytestmark = pytest.mark.gpu

nvq = pytest.importorskip("microscaling_quantized_linear_b200")


SPLIT = [
    # fmt, M, N, K, bias (the library splits K for M <= 32)
    ("nvfp4", 1, 12288, 3072, False),        # FF-up weight at batch 1
    ("nvfp4", 16, 12288, 3072, True),
    ("nvfp4", 32, 9216, 3072, False),        # QKV width
    ("nvfp4", 7, 1000, 2048, True),          # ragged N: the last tile mostly past N
    ("mxfp8", 24, 3072, 12288, True),        # FF-down weight at a short M
    ("mxfp8_e5m2", 3, 2048, 1024, False),
    # shares that do not fall on whole rows or on groups of eight columns
    ("nvfp4", 29, 256, 4096, True),          # 192 wide, split 8, ragged N
    ("nvfp4", 13, 4096, 3072, True),         # 192 wide, split 6
    ("mxfp8", 32, 2048, 3072, False),        # 128 wide, split 6
]


def test_plan_splits_short_m_only():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for fmt, M, N, K, _ in SPLIT:
        tm, tn, ks = nvq.gemm_plan(fmt, M, N, K)
        print(fmt, M, N, K, "->", tm, tn, ks)
        assert tm == 128 and 2 <= ks <= 8 and tn in (128, 192, 256)
        assert -(-N // tn) * ks <= sms
    assert nvq.gemm_plan("nvfp4", 33, 12288, 3072)[2] == 1     # past the rows where a split pays
    assert nvq.gemm_plan("nvfp4", 128, 12288, 3072) == (128, 128, 1)
    assert nvq.gemm_plan("nvfp4", 129, 12288, 3072) == (256, 256, 1)
    assert nvq.gemm_plan("nvfp4", 4608, 12288, 3072) == (256, 256, 1)
    assert nvq.gemm_plan("nvfp4", 1, 256, 256)[2] == 1        # one K tile: nothing to split
    assert nvq.gemm_plan("nvfp4", 128, 37888, 256)[2] == 1    # the tiles already fill the SMs


@pytest.mark.parametrize("fmt,M,N,K,use_bias", SPLIT)
def test_split_k_full_output(fmt, M, N, K, use_bias):
    x = workloads.normal(M, K, seed=300 + M)
    w = workloads.normal(N, K, seed=301 + N % 97, std=0.05)
    b = workloads.bias(N) if use_bias else None
    ldo = (N + 7) // 8 * 8 + (8 if use_bias else 0)
    D = gpu_linear(fmt, x, w, bias=b, ldo=ldo, guard_rows=2)
    full = D.as_strided((M + 2, ldo), (ldo, 1))
    assert torch.isnan(full[:M, N:]).all(), "columns past N were written"
    assert torch.isnan(full[M:]).all(), "rows past M were written"
    check_gemm(D.float().cpu().numpy(), oracle_linear(fmt, x, w, bias=b))


def test_split_k_flux_like_batch1_and_deterministic():
    """The FF-up linear at batch 1 with the FLUX-like activation recipe."""
    x = workloads.activation("ffup", seed=0, M=1)
    w = workloads.weight("ffup")
    a = gpu_linear("nvfp4", x, w)
    b = gpu_linear("nvfp4", x, w)
    assert torch.equal(a, b)
    check_gemm(a.float().cpu().numpy(), oracle_linear("nvfp4", x, w))


EXACT = [
    # fmt, M, N, K, bias
    ("nvfp4", 1, 12288, 3072, True),
    ("nvfp4", 20, 1000, 2048, False),
    ("mxfp8", 32, 3072, 3072, True),
]


def grid_exponents(c):
    return np.floor(np.log2(c)).astype(np.int64)


@pytest.mark.parametrize("fmt,M,N,K,use_bias", EXACT)
def test_split_k_exact_grid_bit_exact(fmt, M, N, K, use_bias):
    assert nvq.gemm_plan(fmt, M, N, K)[2] > 1
    if fmt == "nvfp4":
        # the constant-1.75 rows hold each tensor's amax 10.5 = 2688 / 256:
        # both global scales are 2^-8 and alpha = 2^-16 multiplies exactly
        x, c = workloads.exact_operand(M, K, seed=M + K, top_row=M // 2)
        w, d = workloads.exact_operand(N, K, seed=N + 7, top_row=0)
    else:
        x, c = workloads.exact_operand(M, K, seed=M + K, significands=(1.0, 1.5))
        w, d = workloads.exact_operand(N, K, seed=N + 7, significands=(1.0, 1.5))
    b = workloads.grid_bias(N, seed=N) if use_bias else None
    if fmt == "nvfp4":
        A = oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(bits(x)), M, K)
        B = oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(bits(w)), N, K)
    else:
        A = oracle.mxfp8_dequantize(*oracle.mxfp8_quantize(bits(x)), M, K)
        B = oracle.mxfp8_dequantize(*oracle.mxfp8_quantize(bits(w)), N, K)
    assert np.array_equal(A, x.double().numpy()) and np.array_equal(B, w.double().numpy())
    # Every product is a multiple of u = 2^(i_m + j_n - 6) and so is every
    # bias value; with the sum of |terms| below 2^24 u every partial sum, in
    # any order and any split, is a binary32 number.
    u = np.exp2(grid_exponents(c)[:, None] + grid_exponents(d)[None, :] - 6)
    S = np.abs(A) @ np.abs(B).T
    if b is not None:
        S = S + np.abs(b.double().numpy())[None, :]
        assert np.all(np.exp2(-4) >= u)
    assert np.all(S < 2.0 ** 24 * u)
    Y = oracle.gemm_rows(A, B, bias_bits=None if b is None else bits(b.reshape(1, -1)))
    assert np.all(np.float32(Y) == Y)
    want = oracle.double_to_bf16_array(Y)
    D = gpu_linear(fmt, x, w, bias=b).cpu().view(torch.int16).numpy().view(np.uint16)
    bad = np.argwhere(D != want)
    assert bad.size == 0, "outputs differ at %s" % bad[:8]


SWITCH_SCRIPT = r"""
import microscaling_quantized_linear_b200 as nvq
print(nvq.gemm_plan("nvfp4", 1, 12288, 3072))
"""


def test_split_k_switch_off():
    env = dict(os.environ, NVQ_GEMM_SPLITK="0")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", SWITCH_SCRIPT], env=env, cwd=root,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip().endswith("(128, 128, 1)"), out.stdout
