"""GPU parity of the one-launch short-batch NVFP4 linear (nvfp4_linear_short_m):
the split-K GEMM quantizes the activation itself (each CTA quantizes its own
share of K into its stages; the amax comes from the whole activation up to
4 rows, and above 4 rows from partial maxima the cluster's CTAs exchange).

  * the output equals nvfp4_quantize + block_scaled_linear bit for bit (same
    codes, scales and global scale, same split-K order), and meets the GEMM
    tolerance against the oracle;
  * the optional activation outputs equal the oracle's quantization bit for
    bit (codes, scales with zero padding rows, global scale);
  * pitched input, bias, ragged N; repeated calls replayed from a CUDA graph
    with new activation contents;
  * shapes where the fused launch does not apply return NVQ_ERR_SHAPE and
    launch nothing; a NaN/Inf amax sets NVQ_STATUS_NONFINITE.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import bits, check_gemm

pytestmark = pytest.mark.gpu

nvq = pytest.importorskip("microscaling_quantized_linear_b200")

SHAPES = [
    # M, N, K, bias, pad (pitch = K + pad)
    (1, 12288, 3072, False, 0),     # FF-up weight at batch 1
    (16, 12288, 3072, True, 0),
    (5, 9216, 3072, True, 64),      # QKV width, pitched input
    (3, 1000, 2048, True, 0),       # ragged N
    (16, 3072, 4096, False, 8),
]


def weight(N, K, seed):
    w = workloads.normal(N, K, seed=seed, std=0.05)
    wc, ws, wg = nvq.quantize_weight("nvfp4", w.cuda())
    return w, wc, ws, wg


def activation(M, K, pad, seed):
    x = workloads.normal(M, K, seed=seed)
    x[M // 2, K // 5] = 24.0
    if pad == 0:
        return x, x.cuda()
    buf = torch.zeros(M, K + pad, dtype=torch.bfloat16)
    buf[:, :K] = x
    return x, buf.cuda()[:, :K]


@pytest.mark.parametrize("M,N,K,use_bias,pad", SHAPES)
def test_fused_equals_two_calls_and_the_oracle(M, N, K, use_bias, pad):
    assert nvq.gemm_plan("nvfp4", M, N, K)[2] > 1
    w, wc, ws, wg = weight(N, K, seed=N + K)
    x, xd = activation(M, K, pad, seed=M + 11)
    b = workloads.bias(N) if use_bias else None
    bd = None if b is None else b.cuda()
    ac = torch.full((M, K // 2), 0xA5, dtype=torch.uint8, device="cuda")
    asf = torch.full((nvq.scale_bytes("nvfp4", M, K),), 0xA5, dtype=torch.uint8, device="cuda")
    ag = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    D = nvq.nvfp4_linear_short_m(xd, wc, ws, wg, N, bias=bd, a_codes=ac, a_scales=asf, a_global=ag)
    assert nvq.device_status() == 0
    # the activation's quantization, as the oracle defines it
    oc, osf, og = oracle.nvfp4_quantize(bits(x))
    assert np.array_equal(ac.cpu().numpy(), oc)
    assert np.array_equal(asf.cpu().numpy(), osf)
    assert np.float32(ag.item()).tobytes() == np.float32(og).tobytes()
    # the two-call path, bit for bit
    c2, s2, g2 = nvq.nvfp4_quantize(xd)
    D2 = nvq.block_scaled_linear("nvfp4", c2, s2, g2, wc, ws, wg, M, N, K, bias=bd)
    assert nvq.device_status() == 0
    assert torch.equal(D.view(torch.int16), D2.view(torch.int16))
    A = oracle.nvfp4_dequantize(oc, osf, og, M, K)
    B = oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(bits(w)), N, K)
    Y = oracle.gemm_rows(A, B, bias_bits=None if b is None else bits(b.reshape(1, -1)))
    check_gemm(D.float().cpu().numpy(), Y)


def test_shapes_outside_the_fused_launch_are_refused():
    w, wc, ws, wg = weight(256, 512, seed=3)
    x = torch.zeros(4, 512, dtype=torch.bfloat16, device="cuda")
    # 256 x 512 does not split K (two K stages): NVQ_ERR_SHAPE, nothing launched
    assert nvq.gemm_plan("nvfp4", 4, 256, 512)[2] == 1
    with pytest.raises(nvq.NvqError) as e:
        nvq.nvfp4_linear_short_m(x, wc, ws, wg, 256)
    assert e.value.code == nvq.NVQ_ERR_SHAPE
    w, wc, ws, wg = weight(12288, 3072, seed=4)
    with pytest.raises(nvq.NvqError) as e:
        nvq.nvfp4_linear_short_m(torch.zeros(17, 3072, dtype=torch.bfloat16, device="cuda"), wc, ws, wg, 12288)
    assert e.value.code == nvq.NVQ_ERR_SHAPE
    assert nvq.device_status() == 0


def test_nonfinite_activation_sets_status():
    w, wc, ws, wg = weight(12288, 3072, seed=5)
    x = torch.ones(2, 3072, dtype=torch.bfloat16, device="cuda")
    x[1, 7] = float("inf")
    nvq.nvfp4_linear_short_m(x, wc, ws, wg, 12288)
    assert nvq.device_status() & nvq.NVQ_STATUS_NONFINITE
    assert nvq.device_status() == 0


def test_graph_replays_with_new_activations():
    M, N, K = 1, 12288, 3072
    w, wc, ws, wg = weight(N, K, seed=6)
    B = oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(bits(w)), N, K)
    x_buf = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        x_buf.copy_(workloads.normal(M, K, seed=50).cuda())
        nvq.nvfp4_linear_short_m(x_buf, wc, ws, wg, N, out=out, stream=s)
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            nvq.nvfp4_linear_short_m(x_buf, wc, ws, wg, N, out=out, stream=s)
        s.synchronize()
    for i in range(4):
        x = workloads.normal(M, K, seed=60 + i) * (2.0 ** (4 * i - 6))
        x = x.to(torch.bfloat16)
        with torch.cuda.stream(s):
            x_buf.copy_(x.cuda())
            g.replay()
        s.synchronize()
        assert nvq.device_status() == 0
        A = oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(bits(x)), M, K)
        check_gemm(out.float().cpu().numpy(), oracle.gemm_rows(A, B))
    del g


def test_quantized_linear_takes_the_fused_launch_at_short_batches():
    N, K = 9216, 3072
    w = workloads.normal(N, K, seed=70, std=0.05)
    layer = nvq.QuantizedLinear(w.cuda(), "nvfp4")
    B = oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(bits(w)), N, K)
    for M in (1, 8, 9, 16, 40):
        x = workloads.normal(M, K, seed=M)
        D = layer(x.cuda())
        assert nvq.device_status() == 0
        A = oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(bits(x)), M, K)
        check_gemm(D.float().cpu().numpy(), oracle.gemm_rows(A, B))
    # batches up to SHORT_M_FUSED_ROWS rows took the fused launch, none was refused
    assert nvq.SHORT_M_FUSED_ROWS == 8 and layer._short == {}


def test_waits_run_out_and_the_context_survives():
    # With a 1 ns limit the cluster's exchange of partial maxima and the
    # pipeline waits give up: the amax then comes from the whole activation
    # (exact), the slots still go out, every wait stays bounded, and the host
    # reads NVQ_STATUS_TIMEOUT.  The next call, at the default limit, is clean
    # and equals the two-call path.
    M, N, K = 6, 12288, 3072              # above 4 rows: the cluster exchanges partial maxima
    w, wc, ws, wg = weight(N, K, seed=80)
    x, xd = activation(M, K, 0, seed=81)
    nvq.set_wait_limit(1)
    try:
        for _ in range(3):
            nvq.nvfp4_linear_short_m(xd, wc, ws, wg, N)
        status = nvq.device_status()
    finally:
        nvq.set_wait_limit(0)
    assert status == nvq.NVQ_STATUS_TIMEOUT
    D = nvq.nvfp4_linear_short_m(xd, wc, ws, wg, N)
    assert nvq.device_status() == 0
    c2, s2, g2 = nvq.nvfp4_quantize(xd)
    D2 = nvq.block_scaled_linear("nvfp4", c2, s2, g2, wc, ws, wg, M, N, K)
    assert torch.equal(D.view(torch.int16), D2.view(torch.int16))
