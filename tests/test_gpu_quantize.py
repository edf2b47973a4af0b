"""GPU parity of the quantize kernels against the CPU oracle: bit-exact codes,
block scales and global scale, on every workload's tensors, on ragged and
pitched shapes, and on the special cases."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import act, bits, oracle_nvfp4, sf_matrix, wgt

pytestmark = pytest.mark.gpu

nvq = pytest.importorskip("microscaling_quantized_linear_b200")


def cuda(t):
    return t.to("cuda")


def run_nvfp4(x_cpu, ld=None, calib=None):
    M, K = x_cpu.shape
    if ld is not None and ld != K:
        buf = torch.zeros(M, ld, dtype=torch.bfloat16)
        buf[:, :K] = x_cpu
        xd = cuda(buf)[:, :K]
    else:
        xd = cuda(x_cpu)
    ca = None if calib is None else torch.tensor([calib], dtype=torch.float32, device="cuda")
    codes, sf, g = nvq.nvfp4_quantize(xd, calib_amax=ca)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), sf.cpu().numpy(), np.float32(g.cpu().item())


def run_mxfp8(x_cpu):
    codes, sf = nvq.mxfp8_quantize(cuda(x_cpu))
    torch.cuda.synchronize()
    return codes.cpu().numpy(), sf.cpu().numpy()


def assert_nvfp4_equal(got, want, M, K):
    gc, gs, gg = got
    wc, ws, wg = want
    if not np.array_equal(gc, wc):
        bad = np.argwhere(gc != wc)
        r, b = bad[0]
        raise AssertionError("%d code bytes differ; first at row %d byte %d: gpu %02x oracle %02x"
                             % (len(bad), r, b, gc[r, b], wc[r, b]))
    assert np.array_equal(gs, ws), "%d scale bytes differ" % int((gs != ws).sum())
    assert np.float32(gg).tobytes() == np.float32(wg).tobytes(), (gg, wg)


# ------------------------------------------------------------------ conversion probe

def probe_inputs():
    vals = []
    e4 = [oracle.e4m3_value(c) for c in range(0x7F)]
    e2 = [oracle.e2m1_value(c) for c in range(8)]
    for table in (e4, e2):
        for lo, hi in zip(table[:-1], table[1:]):
            mid = np.float32((lo + hi) / 2)
            vals += [mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e30)),
                     np.float32(lo), np.float32(hi)]
    vals += [0.0, 6.0, 6.5, 7.0, 8.0, 448.0, 464.0, 465.0, 480.0, 1e6, 3e38, 1e-30, 1e-45, 2 ** -10,
             2 ** -9 * 0.5, 2 ** -9 * 0.5001]
    rng = np.random.default_rng(0)
    vals += list((np.float32(2.0) ** rng.uniform(-16, 10, 200000)).astype(np.float32))
    v = np.array(vals, dtype=np.float32)
    return np.concatenate([v, -v])


def test_device_conversions_match_oracle_encoders():
    v = probe_inputs()
    e2, e4 = nvq.probe_convert(torch.from_numpy(v).cuda())
    e2 = e2.cpu().numpy()
    e4 = e4.cpu().numpy()
    want2 = np.array([oracle.e2m1_encode(x) for x in v])
    want4 = np.array([oracle.e4m3_encode(x) for x in v])
    bad2 = np.flatnonzero(e2 != want2)
    bad4 = np.flatnonzero(e4 != want4)
    assert bad2.size == 0, "E2M1 differs at %r: gpu %r oracle %r" % (v[bad2[:5]], e2[bad2[:5]], want2[bad2[:5]])
    assert bad4.size == 0, "E4M3 differs at %r: gpu %r oracle %r" % (v[bad4[:5]], e4[bad4[:5]], want4[bad4[:5]])


# ------------------------------------------------------------------ NVFP4

NVFP4_CASES = [
    ("tiny_act", lambda: act("tiny")),
    ("tiny_w", lambda: workloads.weight("tiny")),
    ("ragged_384x320", lambda: workloads.normal(384, 320, seed=21)),      # 20 blocks per row, 3 row tiles
    ("actq_4608x3072", lambda: act("actq")),
    ("ffup_act", lambda: act("ffup")),
    ("ffup_w_12288x3072", lambda: wgt("ffup")),
    ("qkv4_act_18432x3072", lambda: act("qkv4")),
]


@pytest.mark.parametrize("name,make", NVFP4_CASES, ids=[c[0] for c in NVFP4_CASES])
def test_nvfp4_quantize_bit_exact(name, make):
    x = make()
    M, K = x.shape
    assert_nvfp4_equal(run_nvfp4(x), oracle.nvfp4_quantize(bits(x)), M, K)


def test_nvfp4_quantize_pitched_input():
    x = workloads.normal(256, 448, seed=22)
    assert_nvfp4_equal(run_nvfp4(x, ld=520), oracle.nvfp4_quantize(bits(x)), 256, 448)


def test_nvfp4_calibrated_amax():
    x = act("tiny")
    a = oracle.amax(bits(x))
    for calib in (a, a / 3, a * 5):
        assert_nvfp4_equal(run_nvfp4(x, calib=calib), oracle.nvfp4_quantize(bits(x), calib_amax=calib), 128, 256)


def test_nvfp4_special_tensors():
    cases = {
        "zero": torch.zeros(128, 128, dtype=torch.bfloat16),
        "below_floor": torch.full((128, 64), 2.0 ** -110).to(torch.bfloat16),
        "subnormal_bf16": torch.full((128, 64), 2.0 ** -130).to(torch.bfloat16),
        "neg_zero": torch.full((128, 64), -0.0).to(torch.bfloat16),
        "one_hot": torch.zeros(128, 64).index_put_((torch.tensor([77]), torch.tensor([5])),
                                                   torch.tensor([3.0e38])).to(torch.bfloat16),
    }
    x = workloads.normal(128, 128, seed=23)
    x[3, 16:32] = 0
    x[9, 32:48] = 1e-6        # scale underflows E4M3 -> zero codes
    x[10, 0:16] = -x[10, 0:16].abs()
    cases["mixed_blocks"] = x
    for name, t in cases.items():
        M, K = t.shape
        assert_nvfp4_equal(run_nvfp4(t), oracle.nvfp4_quantize(bits(t)), M, K)


def test_nvfp4_deterministic_and_no_overwrite():
    x = act("ffup")
    M, K = x.shape
    xd = x.cuda()
    guard = 4096
    codes = torch.full((M * K // 2 + 2 * guard,), 0xA5, dtype=torch.uint8, device="cuda")
    sfb = nvq.scale_bytes("nvfp4", M, K)
    sf = torch.full((sfb + 2 * guard,), 0x5A, dtype=torch.uint8, device="cuda")
    g = torch.zeros(4, dtype=torch.float32, device="cuda")
    c_view = codes[guard:guard + M * K // 2].view(M, K // 2)
    s_view = sf[guard:guard + sfb]
    nvq.nvfp4_quantize(xd, c_view, s_view, g[1:2])
    first = (c_view.clone(), s_view.clone(), g.clone())
    nvq.nvfp4_quantize(xd, c_view, s_view, g[1:2])
    torch.cuda.synchronize()
    assert torch.equal(first[0], c_view) and torch.equal(first[1], s_view) and torch.equal(first[2], g)
    assert (codes[:guard] == 0xA5).all() and (codes[-guard:] == 0xA5).all()
    assert (sf[:guard] == 0x5A).all() and (sf[-guard:] == 0x5A).all()
    assert g[0].item() == 0 and g[2].item() == 0
    assert nvq.device_status() == 0


def test_nvfp4_workspace_reuse_across_calls():
    # One workspace for a sequence of different tensors (a zero tensor right
    # after a large one, shapes of different grid sizes): every result must be
    # the oracle's, so no partial maximum of an earlier call can leak into a
    # later one.
    ws = nvq.new_workspace()
    seq = [act("actq"), torch.zeros(4608, 3072, dtype=torch.bfloat16), act("ffup"),
           act("qkv4"), workloads.normal(4608, 3072, seed=77, std=1e-3), act("tiny")]
    for x in seq:
        codes, sf, g = nvq.nvfp4_quantize(x.cuda(), workspace=ws)
        torch.cuda.synchronize()
        M, K = x.shape
        assert_nvfp4_equal((codes.cpu().numpy(), sf.cpu().numpy(), np.float32(g.item())),
                           oracle.nvfp4_quantize(bits(x)), M, K)
    assert nvq.device_status() == 0


def test_nvfp4_nonfinite_input_sets_status():
    nvq.device_status()
    x = workloads.normal(128, 64, seed=3)
    x[7, 7] = float("inf")
    run_nvfp4(x)
    assert nvq.device_status() & nvq.NVQ_STATUS_NONFINITE
    assert nvq.device_status() == 0


def test_empty_batch_launches_nothing():
    x = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    codes, sf, g = nvq.nvfp4_quantize(x)
    c8, s8 = nvq.mxfp8_quantize(x)
    assert codes.numel() == 0 and c8.numel() == 0


ONE_PASS_SCRIPT = r"""
import sys, numpy as np, torch
sys.path.insert(0, ROOT_DIR)
sys.path.insert(0, TEST_DIR)
import test_gpu_quantize as t
import oracle, workloads
import microscaling_quantized_linear_b200 as nvq
from gpu_common import act, bits
ws = nvq.new_workspace()
cases = [act("actq"), act("ffup"), torch.zeros(4608, 3072, dtype=torch.bfloat16),
         workloads.normal(4608, 3072, seed=78, std=1e-3), act("tiny"), workloads.normal(256, 384, seed=31),
         workloads.normal(1152, 6144, seed=79), workloads.normal(100, 3072, seed=81),
         workloads.normal(1000, 1536, seed=82)]
for x in cases:
    codes, sf, g = nvq.nvfp4_quantize(x.cuda(), workspace=ws)
    torch.cuda.synchronize()
    M, K = x.shape
    t.assert_nvfp4_equal((codes.cpu().numpy(), sf.cpu().numpy(), np.float32(g.item())),
                         oracle.nvfp4_quantize(bits(x)), M, K)
    print(M, K, "ok")
assert nvq.device_status() == 0
print("OK")
"""


def test_nvfp4_two_pass_path():
    # The default dynamic NVFP4 quantizer takes one pass (rows held in shared
    # memory) wherever the tensor fits on chip; NVQ_QUANT_ONE_PASS=0 (read
    # when the library loads, hence a fresh process) sends every tensor
    # through the two-pass kernels instead.  Both must give the oracle's
    # results, call after call on one workspace.
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    root = os.path.dirname(here)
    env = dict(os.environ, NVQ_QUANT_ONE_PASS="0")
    script = ONE_PASS_SCRIPT.replace("ROOT_DIR", repr(root)).replace("TEST_DIR", repr(here))
    out = subprocess.run([sys.executable, "-c", script], env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0 and out.stdout.strip().endswith("OK"), out.stdout + out.stderr


def test_nvfp4_one_pass_repeated_calls_and_epochs():
    # the default (one-pass) path, many calls in a row on one workspace:
    # every call's barrier must match only its own epoch
    x = act("ffup")
    ws = nvq.new_workspace()
    want = oracle_nvfp4("ffup", lambda: act("ffup"))
    xd = x.cuda()
    for _ in range(20):
        codes, sf, g = nvq.nvfp4_quantize(xd, workspace=ws)
    torch.cuda.synchronize()
    assert_nvfp4_equal((codes.cpu().numpy(), sf.cpu().numpy(), np.float32(g.item())), want, *x.shape)
    assert nvq.device_status() == 0


# ------------------------------------------------------------------ ragged rows

@pytest.mark.parametrize("M,K", [(1, 256), (100, 3072), (129, 512), (1000, 1536)])
def test_nvfp4_ragged_rows_bit_exact_with_zero_scale_padding(M, K):
    x = workloads.normal(M, K, seed=80 + M)
    codes = torch.full((M, K // 2), 0xA5, dtype=torch.uint8, device="cuda")
    sf = torch.full((nvq.scale_bytes("nvfp4", M, K),), 0xA5, dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    nvq.nvfp4_quantize(x.cuda(), codes, sf, g)
    torch.cuda.synchronize()
    assert_nvfp4_equal((codes.cpu().numpy(), sf.cpu().numpy(), np.float32(g.item())),
                       oracle.nvfp4_quantize(bits(x)), M, K)
    # the calibrated path writes the same padding
    sf2 = torch.full_like(sf, 0x5A)
    ca = torch.tensor([oracle.amax(bits(x))], dtype=torch.float32, device="cuda")
    nvq.nvfp4_quantize(x.cuda(), codes, sf2, g, calib_amax=ca)
    torch.cuda.synchronize()
    assert torch.equal(sf2, sf)
    assert nvq.device_status() == 0


# ------------------------------------------------------------------ MXFP8 variants

def special_mxfp8_tensor():
    """Blocks whose max is exactly 1.75 * 2^e (the rules agree), just above it
    (the ceil rule steps up), BF16 subnormals, values near the BF16 maximum,
    zeros and mixed signs; 128 x 512."""
    x = workloads.normal(128, 512, seed=91).float()
    x[0, :32] *= 1.75 / x[0, :32].abs().max()
    x[1, :32] *= 1.7578125 / x[1, :32].abs().max()
    x[2, 32:64] = x[2, 32:64] * 2.0 ** -130
    x[3, :32] = 3.0e38 * torch.sign(x[3, :32])
    x[4, :64] = 0.0
    x[5, :32] = -x[5, :32].abs()
    x[6, :32] = 57344.0 * 2.0 ** -10
    return x.to(torch.bfloat16)


MXFP8_VARIANTS = [(e, r) for e in ("e4m3", "e5m2") for r in ("floor", "ceil")]
MXFP8_VARIANT_INPUTS = [
    ("tiny_act", lambda: act("tiny")),
    ("ragged_100x384", lambda: workloads.normal(100, 384, seed=33)),
    ("special", special_mxfp8_tensor),
    ("ffdown_act_4608x12288", lambda: act("ffdown")),
]


@pytest.mark.parametrize("elem,rule", MXFP8_VARIANTS, ids=["%s-%s" % v for v in MXFP8_VARIANTS])
@pytest.mark.parametrize("name,make", MXFP8_VARIANT_INPUTS, ids=[c[0] for c in MXFP8_VARIANT_INPUTS])
def test_mxfp8_element_and_rule_variants_bit_exact(elem, rule, name, make):
    x = make()
    M, K = x.shape
    codes = torch.full((M, K), 0xA5, dtype=torch.uint8, device="cuda")
    sf = torch.full((nvq.scale_bytes("mxfp8", M, K),), 0xA5, dtype=torch.uint8, device="cuda")
    nvq.mxfp8_quantize(x.cuda(), codes, sf, elem=elem, rule=rule)
    torch.cuda.synchronize()
    wc, ws = oracle.mxfp8_quantize(bits(x), elem=elem, rule=rule)
    gc = codes.cpu().numpy()
    if not np.array_equal(gc, wc):
        bad = np.argwhere(gc != wc)
        r, k = bad[0]
        raise AssertionError("%d code bytes differ; first at (%d, %d): gpu %02x oracle %02x"
                             % (len(bad), r, k, gc[r, k], wc[r, k]))
    assert np.array_equal(sf.cpu().numpy(), ws), "scale bytes (or their zero padding) differ"


# ------------------------------------------------------------------ MXFP8

MXFP8_CASES = [
    ("tiny_act", lambda: act("tiny")),
    ("ragged_256x384", lambda: workloads.normal(256, 384, seed=31)),
    ("ffdown_act_4608x12288", lambda: act("ffdown")),
    ("ffdown_w_3072x12288", lambda: wgt("ffdown")),
    ("qkv4_act", lambda: act("qkv4")),
]


@pytest.mark.parametrize("name,make", MXFP8_CASES, ids=[c[0] for c in MXFP8_CASES])
def test_mxfp8_quantize_bit_exact(name, make):
    x = make()
    gc, gs = run_mxfp8(x)
    wc, ws = oracle.mxfp8_quantize(bits(x))
    assert np.array_equal(gc, wc), "%d code bytes differ" % int((gc != wc).sum())
    assert np.array_equal(gs, ws), "%d scale bytes differ" % int((gs != ws).sum())


def test_mxfp8_special_tensors():
    x = workloads.normal(128, 256, seed=33)
    x[0, 0:32] = 0
    x[1, 32:64] = 2.0 ** -130            # BF16 subnormals: X clamps to -127
    x[2, 64:96] = 1.8984375              # floor-rule saturation
    x[3, 96:128] = 3.0e38                # largest exponents
    x[4, :] = -0.0
    gc, gs = run_mxfp8(x)
    wc, ws = oracle.mxfp8_quantize(bits(x))
    assert np.array_equal(gc, wc) and np.array_equal(gs, ws)
    S = sf_matrix(gs, 128, 8)
    assert S[0, 0] == 0 and S[2, 2] == 119
