"""GPU parity of QuantizedLinear, the binding's layer object (weight quantized
once, activation quantized on every call, then the block-scaled GEMM): for
each format, full outputs against the oracle's linear over the same
quantization, through repeated calls with different batch sizes (the layer
keeps one activation buffer set per batch size), with and without bias."""
import numpy as np
import pytest

import oracle
import workloads
from gpu_common import bits, check_gemm

pytestmark = pytest.mark.gpu

nvq = pytest.importorskip("microscaling_quantized_linear_b200")

ELEM = {"mxfp8": "e4m3", "mxfp8_e5m2": "e5m2"}


def oracle_linear(fmt, x, w, bias):
    M, K = x.shape
    N = w.shape[0]
    if fmt == "nvfp4":
        A = oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(bits(x)), M, K)
        B = oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(bits(w)), N, K)
    else:
        e = ELEM[fmt]
        A = oracle.mxfp8_dequantize(*oracle.mxfp8_quantize(bits(x), elem=e), M, K, elem=e)
        B = oracle.mxfp8_dequantize(*oracle.mxfp8_quantize(bits(w), elem=e), N, K, elem=e)
    return oracle.gemm_rows(A, B, bias_bits=None if bias is None else bits(bias.reshape(1, -1)))


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp8", "mxfp8_e5m2"])
@pytest.mark.parametrize("use_bias", [False, True])
def test_quantized_linear_matches_oracle(fmt, use_bias):
    N, K = 640, 1024
    w = workloads.normal(N, K, seed=41, std=0.05)
    b = workloads.bias(N) if use_bias else None
    layer = nvq.QuantizedLinear(w.cuda(), fmt, bias=None if b is None else b.cuda())
    for i, M in enumerate((256, 7, 300, 256, 1)):
        x = workloads.normal(M, K, seed=100 + i)
        D = layer(x.cuda())
        assert nvq.device_status() == 0
        assert D.shape == (M, N)
        check_gemm(D.float().cpu().numpy(), oracle_linear(fmt, x, w, b))
