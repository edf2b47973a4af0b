"""GPU parity on seeded random shapes: shapes the hand-picked cases do not
name, drawn from ranges that reach every kernel (the small-tensor cluster
quantizer, the one-pass and two-pass NVFP4 quantizers, MXFP8, one-CTA GEMM
tiles of 128/192/256 columns, CTA pairs, split-K clusters), with ragged rows,
ragged columns and pitched inputs.

Quantizers: codes, scales and the global scale bit-exact against the
oracle.  GEMM: every output within the row-normalised tolerance of the
oracle's binary64 sum of the dequantized operands, NaN canaries past N and
past M untouched.  The draws are fixed by the seed, so a failure reproduces.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import bits, check_gemm
from test_gpu_gemm import gpu_linear, oracle_linear

pytestmark = pytest.mark.gpu

nvq = pytest.importorskip("microscaling_quantized_linear_b200")


def draw_quant_shapes(seed, n):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        M = int(rng.choice([rng.integers(1, 64), rng.integers(64, 700), rng.integers(700, 3000)]))
        K = 64 * int(rng.integers(1, 160))                    # K % 64 == 0, up to 10176
        pad = 8 * int(rng.choice([0, 0, rng.integers(1, 40)]))   # pitch in 16-byte steps
        out.append((M, K, pad))
    return out


def pitched(x, pad):
    if pad == 0:
        return x.cuda()
    M, K = x.shape
    buf = torch.zeros(M, K + pad, dtype=torch.bfloat16)
    buf[:, :K] = x
    return buf.cuda()[:, :K]


@pytest.mark.parametrize("M,K,pad", draw_quant_shapes(2024, 16))
def test_nvfp4_random_shapes_bit_exact(M, K, pad):
    x = workloads.normal(M, K, seed=M * 7 + K)
    x[M // 2, K // 3] = 40.0                                 # an outlier sets the amax
    c, s, g = nvq.nvfp4_quantize(pitched(x, pad))
    assert nvq.device_status() == 0
    oc, osf, og = oracle.nvfp4_quantize(bits(x))
    assert np.array_equal(c.cpu().numpy(), oc), (M, K, pad)
    assert np.array_equal(s.cpu().numpy(), osf), (M, K, pad)
    assert np.float32(g.item()).tobytes() == np.float32(og).tobytes()


@pytest.mark.parametrize("M,K,pad", [(M, K - K % 128 or 128, pad) for M, K, pad in draw_quant_shapes(77, 10)])
def test_mxfp8_random_shapes_bit_exact(M, K, pad):
    x = workloads.normal(M, K, seed=M * 5 + K)
    for elem, rule in (("e4m3", "floor"), ("e5m2", "ceil")):
        c, s = nvq.mxfp8_quantize(pitched(x, pad), elem=elem, rule=rule)
        assert nvq.device_status() == 0
        oc, osf = oracle.mxfp8_quantize(bits(x), elem=elem, rule=rule)
        assert np.array_equal(c.cpu().numpy(), oc), (M, K, pad, elem, rule)
        assert np.array_equal(s.cpu().numpy(), osf), (M, K, pad, elem, rule)


def draw_gemm_shapes(seed, n):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        fmt = ["nvfp4", "mxfp8", "mxfp8_e5m2"][i % 3]
        kstep = 256 if fmt == "nvfp4" else 128
        M = int(rng.choice([rng.integers(1, 33), rng.integers(33, 300), 256 * int(rng.integers(1, 4))]))
        N = 8 * int(rng.integers(1, 1200))
        K = kstep * int(rng.integers(1, 12))
        out.append((fmt, M, N, K, bool(rng.integers(0, 2))))
    return out


@pytest.mark.parametrize("fmt,M,N,K,use_bias", draw_gemm_shapes(31337, 15))
def test_gemm_random_shapes(fmt, M, N, K, use_bias):
    x = workloads.normal(M, K, seed=M + 3 * K)
    w = workloads.normal(N, K, seed=N + 5 * K, std=0.05)
    b = workloads.bias(N) if use_bias else None
    ldo = N + (8 if use_bias else 0)
    print(fmt, M, N, K, "plan", nvq.gemm_plan(fmt, M, N, K))
    D = gpu_linear(fmt, x, w, bias=b, ldo=ldo, guard_rows=1)
    full = D.as_strided((M + 1, ldo), (ldo, 1))
    assert torch.isnan(full[:M, N:]).all(), "columns past N were written"
    assert torch.isnan(full[M:]).all(), "rows past M were written"
    check_gemm(D.float().cpu().numpy(), oracle_linear(fmt, x, w, bias=b))
