"""GPU parity of the fused feed-forward epilogue (block_scaled_linear_gelu_mxfp8):
the linear's BF16 result D goes through GELU and MXFP8 quantization inside
the GEMM, so only the next layer's MXFP8 codes and scales are written.

The oracle composes its definitions: binary64 GEMM over the dequantized
operands, one rounding to BF16, the exact-erf GELU rounded once to BF16, then
MXFP8 (E4M3, floor exponent).  The codes are a function of D alone, and D is
unique only where the GEMM is exact, so:
  * the GELU itself is compared on every one of the 65536 BF16 inputs;
  * on operands drawn on a coarse binary grid (workloads.exact_operand) every
    partial sum of the GEMM is a binary32 number, whatever order the tensor
    core adds in, so D equals the oracle's D and codes and scales must match
    bit for bit (the test first checks that the grid bound holds);
  * on the FLUX-like FF-up workload D is known only to the GEMM tolerance,
    so several results are correct.  From the oracle's Y and the tolerance
    the test derives, for every element, the BF16 values D may take, the
    smallest and largest GELU over them, hence for every 32-block the
    admissible E8M0 exponents and for every element the admissible E4M3
    codes under the exponent the kernel chose; no byte may fall outside
    (check_admissible);
  * the whole feed-forward block (fused FF-up, then the MXFP8 FF-down GEMM
    on its output) meets the GEMM tolerance against the oracle's chain.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from admissible import check_admissible
from gpu_common import act, bits, check_gemm, sample_rows, sf_matrix, wgt

pytestmark = pytest.mark.gpu

nvq = pytest.importorskip("microscaling_quantized_linear_b200")


def test_gelu_probe_all_bf16_inputs():
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = nvq.probe_gelu(torch.from_numpy(allbits.view(np.int16)).cuda()).cpu().numpy().view(np.uint16)
    want = oracle.gelu_bf16_array(allbits)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, ["%04x: gpu %04x oracle %04x" % (i, got[i], want[i]) for i in bad[:10]]


def quantize_both(fmt, x, w):
    """GPU quantization of activation and weight, checked bit-exact against
    the oracle's; returns the GPU operands and the oracle-dequantized ones."""
    M, K = x.shape
    N = w.shape[0]
    xd, wd = x.cuda(), w.cuda()
    if fmt == "nvfp4":
        ac, as_, ag = nvq.nvfp4_quantize(xd)
        wc, ws, wg = nvq.quantize_weight("nvfp4", wd)
        oac, oas, oag = oracle.nvfp4_quantize(bits(x))
        owc, ows, owg = oracle.nvfp4_quantize(bits(w))
        assert np.array_equal(ac.cpu().numpy(), oac) and np.array_equal(as_.cpu().numpy(), oas)
        assert np.array_equal(wc.cpu().numpy(), owc) and np.array_equal(ws.cpu().numpy(), ows)
        assert np.float32(ag.item()) == oag and np.float32(wg.item()) == owg
        A = oracle.nvfp4_dequantize(oac, oas, oag, M, K)
        B = oracle.nvfp4_dequantize(owc, ows, owg, N, K)
    else:
        ac, as_ = nvq.mxfp8_quantize(xd)
        wc, ws, _ = nvq.quantize_weight("mxfp8", wd)
        ag = wg = None
        oac, oas = oracle.mxfp8_quantize(bits(x))
        owc, ows = oracle.mxfp8_quantize(bits(w))
        assert np.array_equal(ac.cpu().numpy(), oac) and np.array_equal(as_.cpu().numpy(), oas)
        assert np.array_equal(wc.cpu().numpy(), owc) and np.array_equal(ws.cpu().numpy(), ows)
        A = oracle.mxfp8_dequantize(oac, oas, M, K)
        B = oracle.mxfp8_dequantize(owc, ows, N, K)
    return (ac, as_, ag, wc, ws, wg), A, B


def gpu_fused(fmt, ops, M, N, K, bias=None):
    ac, as_, ag, wc, ws, wg = ops
    # canary-filled outputs: a byte the kernel fails to write shows up
    yc = torch.full((M, N), 0xA5, dtype=torch.uint8, device="cuda")
    ys = torch.full((nvq.scale_bytes("mxfp8", M, N),), 0xA5, dtype=torch.uint8, device="cuda")
    nvq.block_scaled_linear_gelu_mxfp8(fmt, ac, as_, ag, wc, ws, wg, M, N, K,
                                       bias=None if bias is None else bias.cuda(), y_codes=yc, y_scales=ys)
    assert nvq.device_status() == 0
    return yc.cpu().numpy(), ys.cpu().numpy()


EXACT = [
    # fmt, M, N, K, bias.  The library's tile choice: M > 128 runs CTA pairs
    # on 256 x 256 tiles (rows past M read as zero, the scale rows up to the
    # next multiple of 128 written as zero); M <= 128 one CTA per 128 x 128
    # tile, or 128 x 256 once those tiles fill every SM.
    ("nvfp4", 256, 512, 512, False),
    ("nvfp4", 384, 768, 512, True),       # the last pair tile's second CTA past m_pad
    ("nvfp4", 200, 512, 256, True),       # ragged M
    ("nvfp4", 1024, 1280, 512, False),    # several tiles per CTA pair, N % 256 = 0
    ("nvfp4", 512, 384, 256, True),       # N % 256 = 128: half of the last tile past N
    ("nvfp4", 100, 384, 256, False),      # one CTA, 128 x 128 tiles
    ("nvfp4", 128, 37888, 256, True),     # one CTA, 128 x 256 tiles (148 tiles)
    ("mxfp8", 256, 512, 512, True),
    ("mxfp8", 96, 256, 256, False),
    ("mxfp8", 640, 768, 384, False),
]


def grid_exponents(c):
    return np.floor(np.log2(c)).astype(np.int64)


@pytest.mark.parametrize("fmt,M,N,K,use_bias", EXACT)
def test_exact_grid_bit_exact(fmt, M, N, K, use_bias):
    if fmt == "nvfp4":
        # the row of constant 1.75 holds the tensor's amax 10.5 = 2688 / 256,
        # so both global scales are 2^-8 and alpha = 2^-16 multiplies exactly
        x, c = workloads.exact_operand(M, K, seed=M + K, top_row=M // 2)
        w, d = workloads.exact_operand(N, K, seed=N + 7, top_row=0)
    else:
        # 1.75 * 6 is not an E4M3 multiple of the block's power of two
        x, c = workloads.exact_operand(M, K, seed=M + K, significands=(1.0, 1.5))
        w, d = workloads.exact_operand(N, K, seed=N + 7, significands=(1.0, 1.5))
    b = workloads.grid_bias(N, seed=N) if use_bias else None
    ops, A, B = quantize_both(fmt, x, w)
    assert np.array_equal(A, x.double().numpy()) and np.array_equal(B, w.double().numpy())

    # Every product a(m,k) b(n,k) is a multiple of u = 2^(i_m + j_n - 6)
    # (c = s 2^i with 4s an integer, the e values multiples of 1/2), and so is
    # every bias value (multiples of 1/16, with i, j >= -3).  If the sum of
    # all |terms| stays below 2^24 u, every partial sum in any order, scaled
    # by the power-of-two block scales, is a binary32 number: the tensor
    # core's sum is exact and D = bf16(Y) on both sides.
    u = np.exp2(grid_exponents(c)[:, None] + grid_exponents(d)[None, :] - 6)
    S = np.abs(A) @ np.abs(B).T
    if b is not None:
        S = S + np.abs(b.double().numpy())[None, :]
        assert np.all(np.exp2(-4) >= u)
    assert np.all(S < 2.0 ** 24 * u)

    yc, ys = gpu_fused(fmt, ops, M, N, K, bias=b)
    oc, osf, D, G, Y = oracle.linear_gelu_mxfp8(A, B, bias_bits=None if b is None else bits(b.reshape(1, -1)))
    assert np.all(np.float32(Y) == Y)
    assert ys.size == osf.size
    bad = np.nonzero(ys != osf)[0]
    assert bad.size == 0, "scale bytes differ at %s" % bad[:8]
    badc = np.argwhere(yc != oc)
    assert badc.size == 0, "codes differ at %s" % badc[:8]


def test_exact_grid_deterministic_and_reusable_outputs():
    x, _ = workloads.exact_operand(256, 512, seed=5, top_row=3)
    w, _ = workloads.exact_operand(512, 512, seed=6, top_row=1)
    ops, _, _ = quantize_both("nvfp4", x, w)
    a = gpu_fused("nvfp4", ops, 256, 512, 512)
    b = gpu_fused("nvfp4", ops, 256, 512, 512)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def check_sampled_rows(yc, ys, A, B, rows, M, N):
    """The kernel's outputs on the sampled rows, against the admissible sets."""
    Y = oracle.gemm_rows(A, B, rows=rows)
    check_admissible(yc[rows], sf_matrix(ys, M, N // 32)[rows], Y)
    # every sampled row was written (no canary row left)
    assert not np.all(yc[rows] == 0xA5, axis=1).any()


def test_ffup_workload_sampled_rows():
    """FF-up of the FLUX-like block at full size (4608 x 12288 x 3072, NVFP4),
    in the launch configuration the benchmark uses: every byte of every other
    128-row tile's first and last row (and random rows) admissible."""
    x, w = act("ffup"), wgt("ffup")
    M, K = x.shape
    N = w.shape[0]
    ops, A, B = quantize_both("nvfp4", x, w)
    yc, ys = gpu_fused("nvfp4", ops, M, N, K)
    check_sampled_rows(yc, ys, A, B, sample_rows(M, per_tile_every=2, extra=16), M, N)


def test_feed_forward_block_end_to_end():
    """Fused FF-up (NVFP4, GELU, MXFP8 out), then the MXFP8 FF-down GEMM on
    its output, against the oracle's chain (the FF-down operand is the
    oracle's own MXFP8 quantization of its GELU output)."""
    M, H, F = 512, 1024, 2048
    x = workloads.activation("ffup", seed=9, M=M, K=H)
    w1 = workloads.weight("ffup", seed=10, N=F, K=H)
    w2 = workloads.weight("ffdown", seed=11, N=H, K=F)
    ops, A, B = quantize_both("nvfp4", x, w1)
    yc = torch.empty((M, F), dtype=torch.uint8, device="cuda")
    ys = torch.empty(nvq.scale_bytes("mxfp8", M, F), dtype=torch.uint8, device="cuda")
    ac, as_, ag, wc, ws, wg = ops
    nvq.block_scaled_linear_gelu_mxfp8("nvfp4", ac, as_, ag, wc, ws, wg, M, F, H, y_codes=yc, y_scales=ys)
    w2c, w2s, _ = nvq.quantize_weight("mxfp8", w2.cuda())
    out = nvq.block_scaled_linear("mxfp8", yc, ys, None, w2c, w2s, None, M, H, F)
    assert nvq.device_status() == 0
    oc, osf, _, _, _ = oracle.linear_gelu_mxfp8(A, B)
    o2c, o2s = oracle.mxfp8_quantize(bits(w2))
    Y2 = oracle.gemm_rows(oracle.mxfp8_dequantize(oc, osf, M, F), oracle.mxfp8_dequantize(o2c, o2s, H, F))
    check_gemm(out.float().cpu().numpy(), Y2)


def test_ffup_workload_mxfp8_operands_sampled_rows():
    """The same FF-up linear with MXFP8 (E4M3) activation and weight operands."""
    x, w = act("ffup"), wgt("ffup")
    M, K = x.shape
    N = w.shape[0]
    ops, A, B = quantize_both("mxfp8", x, w)
    yc, ys = gpu_fused("mxfp8", ops, M, N, K)
    check_sampled_rows(yc, ys, A, B, sample_rows(M, per_tile_every=2, extra=8), M, N)


SINGLE_CTA_FUSED_SCRIPT = r"""
import sys, numpy as np
sys.path.insert(0, ROOT_DIR)
sys.path.insert(0, TEST_DIR)
import test_gpu_fused as t
import workloads, oracle
from gpu_common import bits, sample_rows
# exact-grid operands: bit-exact codes and scales through the one-CTA kernel
for fmt, M, N, K in [("nvfp4", 512, 768, 512), ("nvfp4", 1280, 512, 256), ("mxfp8", 384, 512, 256)]:
    if fmt == "nvfp4":
        x, _ = workloads.exact_operand(M, K, seed=M + 3, top_row=1)
        w, _ = workloads.exact_operand(N, K, seed=N + 5, top_row=2)
    else:
        x, _ = workloads.exact_operand(M, K, seed=M + 3, significands=(1.0, 1.5))
        w, _ = workloads.exact_operand(N, K, seed=N + 5, significands=(1.0, 1.5))
    ops, A, B = t.quantize_both(fmt, x, w)
    yc, ys = t.gpu_fused(fmt, ops, M, N, K)
    oc, osf, _, _, _ = oracle.linear_gelu_mxfp8(A, B)
    assert np.array_equal(ys, osf) and np.array_equal(yc, oc), (fmt, M, N, K)
    print(fmt, M, N, K, "bit-exact")
# the FF-up workload, NVFP4 and MXFP8 operands: every byte admissible on the
# sampled rows of every other 128-row tile
x, w = t.act("ffup"), t.wgt("ffup")
M, K = x.shape
N = w.shape[0]
for fmt in ("nvfp4", "mxfp8"):
    ops, A, B = t.quantize_both(fmt, x, w)
    yc, ys = t.gpu_fused(fmt, ops, M, N, K)
    t.check_sampled_rows(yc, ys, A, B, sample_rows(M, per_tile_every=2, extra=8), M, N)
    print(fmt, "FF-up admissible")
print("OK")
"""


def test_single_cta_kernel_fused_epilogue():
    # NVQ_GEMM_PAIRS=0 (read when the library loads, hence a fresh process)
    # sends every shape through the one-CTA kernel with the fused epilogue
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    root = os.path.dirname(here)
    env = dict(os.environ, NVQ_GEMM_PAIRS="0")
    script = SINGLE_CTA_FUSED_SCRIPT.replace("ROOT_DIR", repr(root)).replace("TEST_DIR", repr(here))
    out = subprocess.run([sys.executable, "-c", script], env=env, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0 and out.stdout.strip().endswith("OK"), out.stdout + out.stderr
