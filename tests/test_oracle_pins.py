"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test pins a part of the oracle to a library routine, a closed form, a
value printed on the pages, a hand-worked example, an invariant or brute
force, so that a plausible slip in the oracle (a dropped term, a wrong sign
or index, a swapped nibble, a transposed operand) fails at least one of them.
"""
import json
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
import workloads


def bits(x_bf16):
    return x_bf16.contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16(vals, shape=None):
    t = torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)
    return t.reshape(shape) if shape else t


# --------------------------------------------------------------------------
# Element formats against library decoders (torch / ml_dtypes)
# --------------------------------------------------------------------------

def test_e2m1_decode_matches_ml_dtypes():
    lib_vals = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    ours = np.array([oracle.e2m1_value(c) for c in range(16)])
    assert np.array_equal(np.signbit(ours), np.signbit(lib_vals))
    assert np.array_equal(ours, lib_vals)


def test_e4m3_decode_matches_torch_all_256_codes():
    lib_vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    ours = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(lib_vals)
    assert np.array_equal(np.isnan(ours), nan)
    assert set(np.flatnonzero(nan)) == {0x7F, 0xFF}
    assert np.array_equal(ours[~nan], lib_vals[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(lib_vals[~nan]))
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def test_e8m0_decode_matches_torch_all_256_codes():
    lib_vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    ours = np.array([oracle.e8m0_value(c) for c in range(256)])
    assert np.isnan(ours[255]) and np.isnan(lib_vals[255])
    assert np.array_equal(ours[:255], lib_vals[:255])


def test_encode_decode_round_trip_every_finite_code():
    for c in range(16):
        assert oracle.e2m1_encode(oracle.e2m1_value(c)) == c
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert oracle.e4m3_encode(oracle.e4m3_value(c)) == c, hex(c)


def _torch_e4m3_code(v):
    t = torch.tensor(np.asarray(v, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy().astype(np.int64)


def test_e4m3_encode_midpoints_and_neighbours_match_torch():
    # Every pair of adjacent non-negative values: the midpoint and one FP32 ulp
    # either side, both signs.  torch's float8_e4m3fn cast is round-to-nearest
    # -even; above 448 it returns NaN instead of saturating, so stay below 464.
    vals = [oracle.e4m3_value(c) for c in range(0x7F)]
    probes = []
    for lo, hi in zip(vals[:-1], vals[1:]):
        mid = np.float32((lo + hi) / 2)
        probes += [mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9))]
    probes = np.array(probes, dtype=np.float32)
    probes = np.concatenate([probes, -probes])
    ours = np.array([oracle.e4m3_encode(v) for v in probes])
    assert np.array_equal(ours, _torch_e4m3_code(probes))


def test_e4m3_encode_random_matches_torch():
    rng = np.random.default_rng(7)
    mag = np.float32(2.0) ** rng.uniform(-14, 8.85, 20000).astype(np.float32)
    v = (mag * rng.choice([-1, 1], mag.size)).astype(np.float32)
    v = v[np.abs(v) < 464]
    ours = np.array([oracle.e4m3_encode(x) for x in v])
    assert np.array_equal(ours, _torch_e4m3_code(v))


def test_e4m3_encode_array_matches_torch_and_saturates():
    # The array form: every midpoint +- 1 ulp and random values against
    # torch's RNE cast (below 464), then saturation, infinities and -0.
    vals = [oracle.e4m3_value(c) for c in range(0x7F)]
    probes = []
    for lo, hi in zip(vals[:-1], vals[1:]):
        mid = np.float32((lo + hi) / 2)
        probes += [mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9)), lo]
    rng = np.random.default_rng(11)
    probes += list(np.float32(2.0) ** rng.uniform(-20, 8.85, 20000).astype(np.float32))
    p = np.array(probes, dtype=np.float32)
    p = np.concatenate([p, -p])
    assert np.array_equal(oracle.e4m3_encode_array(p).astype(np.int64), _torch_e4m3_code(p))
    big = np.array([448.0, 464.0, 486.4, 1e6, np.inf, -np.inf, -0.0, -1e-9], dtype=np.float32)
    assert oracle.e4m3_encode_array(big).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x80, 0x80]


def test_e4m3_saturation():
    assert oracle.e4m3_encode(448.0) == 0x7E
    assert oracle.e4m3_encode(464.0) == 0x7E       # tie with the missing 480 -> even 0x7E
    assert oracle.e4m3_encode(486.4) == 0x7E
    assert oracle.e4m3_encode(1e6) == 0x7E
    assert oracle.e4m3_encode(-1e30) == 0xFE
    assert oracle.e4m3_encode(-1e-9) == 0x80       # rounds to zero, sign kept


def test_e2m1_encode_matches_ml_dtypes():
    # ml_dtypes' float4_e2m1fn cast rounds to nearest even and saturates at 6.
    rng = np.random.default_rng(3)
    grid = np.arange(0, 8.0, 0.125, dtype=np.float32)          # every tie and beyond 6
    v = np.concatenate([grid, -grid, rng.normal(0, 3, 5000).astype(np.float32),
                        np.array([6.2222223, 7.0, 100.0, -0.1, -0.0], dtype=np.float32)])
    lib_codes = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    ours = np.array([oracle.e2m1_encode(x) for x in v])
    assert np.array_equal(ours, lib_codes)


def test_e2m1_ties_go_to_even_code():
    expect = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for v, c in expect.items():
        assert oracle.e2m1_encode(v) == c
        assert oracle.e2m1_encode(-v) == c | 0x8


def test_nan_input_is_flagged():
    oracle.take_nan_flag()
    oracle.e4m3_encode(float("nan"))
    assert oracle.take_nan_flag()
    assert not oracle.take_nan_flag()


# --------------------------------------------------------------------------
# Values printed on the pages, and hand-worked blocks
# --------------------------------------------------------------------------

def test_page5_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "page5_worked_example.json")))
    ratio = np.float32(g["x"]) / np.float32(g["scale"])
    code = oracle.e4m3_encode(ratio)
    assert code == g["e4m3_code"]
    assert oracle.e4m3_value(code) == g["q"]
    assert abs(oracle.e4m3_value(code) * g["scale"] - g["x_dequant"]) < 1e-12


def test_nvfp4_hand_worked_blocks(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "nvfp4_hand_blocks.json")))
    x = bf16(g["x"], (g["rows"], g["K"]))
    codes, sf, gdec = oracle.nvfp4_quantize(bits(x))
    assert codes.tobytes().hex() == g["codes_hex"]
    nblk = g["K"] // 16
    assert [int(sf[oracle.sf_offset(0, j, nblk)]) for j in range(nblk)] == g["scale_codes"]
    assert np.float32(gdec).tobytes()[::-1].hex() == g["g_dec_hex"]


def test_mxfp8_hand_worked_blocks(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "mxfp8_hand_blocks.json")))
    vals = np.zeros(g["K"], dtype=np.float32)
    for k, v in g["x_block0"].items():
        vals[int(k)] = v
    for k, v in g["x_block1"].items():
        vals[32 + int(k)] = v
    x = bf16(vals.tolist(), (1, g["K"]))
    codes, sf = oracle.mxfp8_quantize(bits(x))
    assert [int(sf[oracle.sf_offset(0, j, 2)]) for j in range(2)] == g["scale_codes"]
    for key, c in g["codes"].items():
        b, i = map(int, key.split(":"))
        assert int(codes[0, 32 * b + i]) == c


def test_nvfp4_storage_ratio_page1():
    # Page 1, NVFP4: about 3.5x less memory than BF16 (4-bit values + one
    # 8-bit scale per 16 values).
    x = workloads.normal(256, 1024, seed=5)
    codes, sf, _ = oracle.nvfp4_quantize(bits(x))
    ratio = (2 * x.numel()) / (codes.nbytes + sf.nbytes)
    assert abs(ratio - 16 / 4.5) < 1e-9 and 3.4 < ratio < 3.6


# --------------------------------------------------------------------------
# Special cases
# --------------------------------------------------------------------------

def test_zero_tensor_nvfp4():
    x = torch.zeros(128, 64, dtype=torch.bfloat16)
    codes, sf, g = oracle.nvfp4_quantize(bits(x))
    assert g == 0 and not codes.any() and not sf.any()


def test_tiny_tensor_below_floor_is_zero():
    x = bf16([2.0 ** -110] * 64, (1, 64))
    codes, sf, g = oracle.nvfp4_quantize(bits(x))
    assert g == 0 and not codes.any() and not sf.any()
    x = bf16([2.0 ** -99] * 64, (1, 64))
    codes, sf, g = oracle.nvfp4_quantize(bits(x))
    assert g > 0 and codes.any()


def test_zero_block_inside_nonzero_tensor():
    x = workloads.normal(128, 64, seed=11)
    x[5, 16:32] = 0
    codes, sf, g = oracle.nvfp4_quantize(bits(x))
    assert sf[oracle.sf_offset(5, 1, 4)] == 0
    assert not codes[5, 8:16].any()
    cm, sm = oracle.mxfp8_quantize(bits(torch.cat([x, x], 1)))
    x2 = torch.cat([x, x], 1)
    x2[7, 32:64] = 0
    cm, sm = oracle.mxfp8_quantize(bits(x2))
    assert sm[oracle.sf_offset(7, 1, 4)] == 0 and not cm[7, 32:64].any()


def test_zero_tensor_mxfp8():
    codes, sf = oracle.mxfp8_quantize(bits(torch.zeros(128, 64, dtype=torch.bfloat16)))
    assert not codes.any()
    nblk = 2
    assert all(sf[oracle.sf_offset(r, j, nblk)] == 0 for r in range(128) for j in range(nblk))


def test_e4m3_scale_underflow_gives_zero_codes():
    # One block holds the tensor max; another is so small that its scale
    # (b/6 * g_enc) is below half the smallest E4M3 subnormal.
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 0] = 1000.0
    x[0, 16] = 1e-4
    codes, sf, g = oracle.nvfp4_quantize(bits(bf16(x.tolist())))
    assert sf[oracle.sf_offset(0, 1, 2)] == 0 and codes[0, 8:16].sum() == 0


def test_calibrated_amax():
    x = workloads.activation("tiny")
    xb = bits(x)
    a = oracle.amax(xb)
    c0, s0, g0 = oracle.nvfp4_quantize(xb)
    c1, s1, g1 = oracle.nvfp4_quantize(xb, calib_amax=a)
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1) and g0 == g1
    # A calibrated range below the live maximum saturates the largest block.
    c2, s2, g2 = oracle.nvfp4_quantize(xb, calib_amax=a / 4)
    r, k = np.unravel_index(np.abs(x.float().numpy()).argmax(), x.shape)
    assert s2[oracle.sf_offset(r, k // 16, x.shape[1] // 16)] == 0x7E
    q = (c2[r, k // 2] >> (4 * (k % 2))) & 0x7
    assert q == 7


# --------------------------------------------------------------------------
# Invariants
# --------------------------------------------------------------------------

@pytest.mark.parametrize("k", [3, -5])
def test_nvfp4_power_of_two_equivariance(k):
    x = workloads.activation("tiny")
    c0, s0, g0 = oracle.nvfp4_quantize(bits(x))
    c1, s1, g1 = oracle.nvfp4_quantize(bits((x.float() * 2.0 ** k).to(torch.bfloat16)))
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1)
    assert g1 == np.float32(g0 * np.float32(2.0 ** k))


@pytest.mark.parametrize("k", [4, -6])
def test_mxfp8_power_of_two_equivariance(k):
    x = workloads.normal(128, 256, seed=9)
    c0, s0 = oracle.mxfp8_quantize(bits(x))
    c1, s1 = oracle.mxfp8_quantize(bits((x.float() * 2.0 ** k).to(torch.bfloat16)))
    assert np.array_equal(c0, c1)
    nblk = 256 // 32
    for r in range(128):
        for j in range(nblk):
            o = oracle.sf_offset(r, j, nblk)
            assert int(s1[o]) == int(s0[o]) + k


def test_sign_symmetry():
    x = workloads.activation("tiny")
    c0, s0, g0 = oracle.nvfp4_quantize(bits(x))
    c1, s1, g1 = oracle.nvfp4_quantize(bits(-x))
    assert np.array_equal(c1, c0 ^ 0x88) and np.array_equal(s0, s1) and g0 == g1
    m0, t0 = oracle.mxfp8_quantize(bits(x))
    m1, t1 = oracle.mxfp8_quantize(bits(-x))
    assert np.array_equal(m1, m0 ^ 0x80) and np.array_equal(t0, t1)


def test_block_locality_and_blocks_run_along_k():
    x = workloads.normal(128, 64, seed=13)
    x[0, 0] = 50.0                                   # fix the tensor amax
    c0, s0, _ = oracle.nvfp4_quantize(bits(x))
    # Permute inside block (row 3, block 2): codes permute, scale unchanged.
    perm = torch.randperm(16, generator=torch.Generator().manual_seed(0))
    y = x.clone()
    y[3, 32:48] = x[3, 32:48][perm]
    c1, s1, _ = oracle.nvfp4_quantize(bits(y))
    nib = lambda c, r, k: (c[r, k // 2] >> (4 * (k % 2))) & 0xF
    assert [nib(c1, 3, 32 + i) for i in range(16)] == [nib(c0, 3, 32 + int(p)) for p in perm]
    assert np.array_equal(s0, s1)
    # Change one block: only its 8 code bytes and its scale byte move.
    y = x.clone()
    y[7, 16:32] = -3 * x[7, 16:32]
    c2, s2, _ = oracle.nvfp4_quantize(bits(y))
    diff = np.argwhere(c2 != c0)
    assert diff.size and all(r == 7 and 8 <= b < 16 for r, b in diff)
    sdiff = np.flatnonzero(s2 != s0)
    assert set(sdiff) <= {oracle.sf_offset(7, 1, 4)}


def test_e2m1_choice_is_nearest_code_brute_force():
    # For every element, the chosen code is the argmin over all 16 codes of
    # |x * r - value(code)| (ties to the even code), with r = g_enc / scale.
    x = workloads.activation("tiny")
    xb = bits(x)
    codes, sf, gdec = oracle.nvfp4_quantize(xb)
    amax = np.float32(oracle.amax(xb))
    g_enc = np.float32(2688.0) / amax
    xf = x.float().numpy()
    table = np.array([oracle.e2m1_value(c) for c in range(16)])
    K = xf.shape[1]
    for m in range(0, 128, 9):
        for j in range(K // 16):
            sv = np.float32(oracle.e4m3_value(sf[oracle.sf_offset(m, j, K // 16)]))
            if sv == 0:
                continue
            r = g_enc / sv
            for i in range(16):
                k = 16 * j + i
                v = np.float64(np.float32(xf[m, k]) * r)
                d = np.abs(table[:8] - min(abs(v), 6.0))
                best = np.flatnonzero(d == d.min())
                want = best[0] if best.size == 1 else [b for b in best if b % 2 == 0][0]
                q = (codes[m, k // 2] >> (4 * (k % 2))) & 0xF
                assert q & 7 == want and (q >> 3) == (1 if np.signbit(v) else 0)


def test_block_scale_maps_block_max_near_six():
    # The decode scale times 6 reproduces the block maximum to E4M3 precision.
    x = workloads.activation("actq", M=128, K=512)
    xb = bits(x)
    codes, sf, gdec = oracle.nvfp4_quantize(xb)
    xf = np.abs(x.float().numpy())
    for m in range(128):
        for j in range(32):
            b = xf[m, 16 * j:16 * j + 16].max()
            sc = sf[oracle.sf_offset(m, j, 32)]
            s = oracle.e4m3_value(sc)
            if sc >= 0x08 and sc < 0x7E:              # normal E4M3, not saturated
                assert abs(6 * s * gdec - b) <= b * 2 ** -4 + 1e-30


# --------------------------------------------------------------------------
# Scale layout
# --------------------------------------------------------------------------

@pytest.mark.parametrize("rows,cols", [(128, 4), (256, 8), (384, 12), (130, 5)])
def test_sf_offset_is_a_bijection(rows, cols):
    n = oracle.sf_bytes(rows, cols)
    rp, cp = -(-rows // 128) * 128, -(-cols // 4) * 4
    assert n == rp * cp
    offs = [oracle.sf_offset(r, c, cols) for r in range(rp) for c in range(cp)]
    assert sorted(offs) == list(range(n))


def test_sf_offset_matches_tensor_permutation():
    # The same layout written as a reshape/transpose of the logical scale
    # matrix: [R/128, 4, 32, C/4, 4] -> [R/128, C/4, 32, 4, 4].
    R, C = 256, 12
    S = np.arange(R * C).reshape(R, C)
    blocked = S.reshape(R // 128, 4, 32, C // 4, 4).transpose(0, 3, 2, 1, 4).reshape(-1)
    ours = np.empty(R * C, dtype=np.int64)
    for r in range(R):
        for c in range(C):
            ours[oracle.sf_offset(r, c, C)] = S[r, c]
    assert np.array_equal(ours, blocked)


# --------------------------------------------------------------------------
# Dequantization and GEMM
# --------------------------------------------------------------------------

def test_nvfp4_dequantize_matches_library_decode():
    x = workloads.activation("tiny")
    codes, sf, g = oracle.nvfp4_quantize(bits(x))
    M, K = x.shape
    got = oracle.nvfp4_dequantize(codes, sf, g, M, K)
    lo = (codes & 0xF).astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    hi = (codes >> 4).astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    e2m1 = np.stack([lo, hi], axis=-1).reshape(M, K)
    S = np.array([[sf[oracle.sf_offset(m, j, K // 16)] for j in range(K // 16)] for m in range(M)],
                 dtype=np.uint8)
    Sv = torch.from_numpy(S).view(torch.float8_e4m3fn).double().numpy()
    want = e2m1 * np.repeat(Sv, 16, axis=1) * np.float64(g)
    assert np.array_equal(got, want)


def test_mxfp8_dequantize_matches_library_decode():
    x = workloads.normal(128, 256, seed=17)
    codes, sf = oracle.mxfp8_quantize(bits(x))
    M, K = x.shape
    got = oracle.mxfp8_dequantize(codes, sf, M, K)
    e4 = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    S = np.array([[sf[oracle.sf_offset(m, j, K // 32)] for j in range(K // 32)] for m in range(M)],
                 dtype=np.uint8)
    Sv = torch.from_numpy(S).view(torch.float8_e8m0fnu).double().numpy()
    assert np.array_equal(got, e4 * np.repeat(Sv, 32, axis=1))


def test_quantization_error_is_small():
    # Round trip error relative to the row norm: loose sanity bound only.
    x = workloads.activation("ffup", M=128, K=512)
    codes, sf, g = oracle.nvfp4_quantize(bits(x))
    xh = oracle.nvfp4_dequantize(codes, sf, g, 128, 512)
    xf = x.double().numpy()
    rel = np.linalg.norm(xh - xf, axis=1) / np.linalg.norm(xf, axis=1)
    assert rel.max() < 0.15
    c8, s8 = oracle.mxfp8_quantize(bits(x))
    x8 = oracle.mxfp8_dequantize(c8, s8, 128, 512)
    # MXFP8 rows with a x50 outlier can lose up to 1/8 of it: under the floor
    # scale rule a block maximum in [448, 512) * 2^X saturates to 448 * 2^X.
    assert (np.linalg.norm(x8 - xf, axis=1) / np.linalg.norm(xf, axis=1)).max() < 0.15


def test_gemm_rows_matches_numpy_matmul():
    rng = np.random.default_rng(1)
    A = rng.normal(size=(37, 96))
    B = rng.normal(size=(20, 96))
    rows = np.array([0, 5, 36, 12])
    out = oracle.gemm_rows(A, B, rows)
    want = A[rows] @ B.T
    assert np.allclose(out, want, rtol=1e-12, atol=1e-12)
    bias = bits(bf16(rng.normal(size=20).tolist()))
    outb = oracle.gemm_rows(A, B, rows, bias_bits=bias)
    bias_f = torch.from_numpy(bias.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.allclose(outb, want + bias_f[None, :], rtol=1e-12, atol=1e-12)


def test_gemm_rows_brute_force_exact_on_integers():
    A = np.array([[1, 2, 0, -1], [3, 0, 1, 1]], dtype=np.float64)
    B = np.array([[1, 0, 0, 0], [0, 1, 0, 0], [2, 2, 2, 2]], dtype=np.float64)
    out = oracle.gemm_rows(A, B)
    assert out.tolist() == [[1, 2, 4], [3, 0, 10]]


def test_acceptance_rule():
    # The output is judged before its BF16 rounding: the error of a BF16
    # output is the distance from Y to the values that round to it.
    Y = np.array([[3.0, 4.0], [0.0, 0.0]])
    assert oracle.gemm_row_errors(Y, Y).tolist() == [0.0, 0.0]
    # 3 + 1/64 is the BF16 neighbour of 3 (spacing 1/64 in [2, 4)): the
    # values that round to it start half a spacing below it, at 3 + 1/128
    D = np.array([[3.015625, 4.0], [0.0, 0.0]])
    assert oracle.gemm_row_errors(D, Y)[0] == 0.0078125 / 5.0
    # at a power of two the spacing below (1/64) is half the spacing above
    # (1/32): 4 covers [4 - 1/128, 4 + 1/64]; mirrored for -4
    assert oracle.gemm_row_errors(np.array([[4.0, 0.0]]), np.array([[4.015, 0.0]]))[0] == 0.0
    assert oracle.gemm_row_errors(np.array([[4.0, 0.0]]), np.array([[4.0165, 0.0]]))[0] > 0.0
    assert oracle.gemm_row_errors(np.array([[-4.0, 0.0]]), np.array([[-4.015, 0.0]]))[0] == 0.0
    err = oracle.gemm_row_errors(np.array([[4.0, 0.0]]), np.array([[3.99, 0.0]]))[0]
    assert abs(err - (3.9921875 - 3.99) / 3.99) < 1e-15
    # an all-zero reference row takes +-0 only; the smallest subnormal is wrong
    D = np.array([[0.0, -0.0], [2.0 ** -133, 0.0]])
    assert oracle.gemm_row_errors(D, np.zeros((2, 2))).tolist() == [0.0, np.inf]
    assert np.isinf(oracle.gemm_row_errors(np.array([[np.inf, 4.0]]), np.array([[3.0, 4.0]]))[0])
    with pytest.raises(AssertionError):
        oracle.gemm_row_errors(np.array([[3.005, 4.0]]), Y[:1])      # not a BF16 value


def test_acceptance_rule_accepts_every_correctly_rounded_output():
    # D = the BF16 rounding of the exact sum is correct for any shape, short
    # rows included: a row whose norm one element carries can lose up to
    # 2^-8 of it to BF16 rounding alone, more than the 2e-3 budget.
    rng = np.random.default_rng(8)
    for n in (1, 2, 3, 24, 257):
        Y = rng.standard_normal((64, n)) * np.exp2(rng.integers(-20, 20, (64, 1)))
        Y[0, 0] = 1.0 + 2.0 ** -8 - 2.0 ** -40     # rounds down to 1 (relative error just under 2^-8)
        D = (oracle.double_to_bf16_array(Y).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        assert np.all(oracle.gemm_row_errors(D, Y) == 0.0), n
        if n == 1:      # |D - Y| itself is above the budget there
            assert abs(D[0, 0] - Y[0, 0]) / abs(Y[0, 0]) > 2e-3


# --------------------------------------------------------------------------
# MXFP8 with E5M2 elements and the ceil block exponent; ragged row counts
# --------------------------------------------------------------------------

def test_e5m2_decode_matches_torch_all_256_codes():
    lib_vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e5m2).double().numpy()
    ours = np.array([oracle.e5m2_value(c) for c in range(256)])
    assert np.array_equal(np.isnan(ours), np.isnan(lib_vals))
    fin = ~np.isnan(lib_vals)
    assert np.array_equal(ours[fin], lib_vals[fin])
    assert np.array_equal(np.signbit(ours[fin]), np.signbit(lib_vals[fin]))
    assert ours[0x7B] == 57344.0 and np.isinf(ours[0x7C]) and ours[0x01] == 2.0 ** -16


def test_e5m2_encode_matches_torch_below_the_maximum():
    # torch's float8_e5m2 cast rounds to nearest even and overflows to inf
    # past the top, so compare at every midpoint +-1 ulp below 57344 and on
    # random values; saturation is checked separately.
    vals = [oracle.e5m2_value(c) for c in range(0x7C)]
    probes = []
    for lo, hi in zip(vals[:-1], vals[1:]):
        mid = np.float32((lo + hi) / 2)
        probes += [mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9))]
    rng = np.random.default_rng(7)
    probes += list((rng.standard_normal(20000) * np.exp2(rng.integers(-18, 15, 20000))).astype(np.float32))
    probes = np.array([p for p in probes if abs(p) < 57344], dtype=np.float32)
    probes = np.concatenate([probes, -probes])
    want = torch.tensor(probes).to(torch.float8_e5m2).view(torch.uint8).numpy().astype(np.int64)
    got = np.array([oracle.e5m2_encode(p) for p in probes])
    assert np.array_equal(got, want)
    for c in range(256):
        if (c & 0x7F) >= 0x7C:
            continue
        assert oracle.e5m2_encode(oracle.e5m2_value(c)) == c, hex(c)
    assert oracle.e5m2_encode(60000.0) == 0x7B and oracle.e5m2_encode(-1e30) == 0xFB


@pytest.mark.parametrize("case", ["e4m3/floor", "e4m3/ceil", "e5m2/floor", "e5m2/ceil"])
def test_mxfp8_element_and_rule_hand_worked_blocks(golden_dir, case):
    g = json.load(open(os.path.join(golden_dir, "mxfp8_elem_rule_blocks.json")))
    vals = np.zeros(g["K"], dtype=np.float32)
    for k, v in g["x_block0"].items():
        vals[int(k)] = v
    for k, v in g["x_block1"].items():
        vals[32 + int(k)] = v
    x = bf16(vals.tolist(), (1, g["K"]))
    assert torch.equal(x.float()[0], torch.tensor(vals))          # the inputs are exact BF16
    elem, rule = case.split("/")
    codes, sf = oracle.mxfp8_quantize(bits(x), elem=elem, rule=rule)
    want = g["cases"][case]
    assert [int(sf[oracle.sf_offset(0, j, 2)]) for j in range(2)] == want["scale_codes"]
    for key, c in want["codes"].items():
        b, i = map(int, key.split(":"))
        assert int(codes[0, 32 * b + i]) == c, (key, hex(int(codes[0, 32 * b + i])), hex(c))


@pytest.mark.parametrize("elem,maxv", [("e4m3", 448.0), ("e5m2", 57344.0)])
def test_mxfp8_block_exponent_rules_by_brute_force(elem, maxv):
    # floor rule: X = floor(log2 b) - emax, from the exact binary exponent;
    # ceil rule: the smallest integer X with b <= max * 2^X, by search over X.
    emax = 8 if elem == "e4m3" else 15
    x = workloads.normal(64, 256, seed=23, std=3.0)
    x[3, :32] *= 1e-30
    xb = x.float().numpy()
    for rule in ("floor", "ceil"):
        _, sf = oracle.mxfp8_quantize(bits(x), elem=elem, rule=rule)
        for r in range(64):
            for j in range(8):
                b = float(np.abs(xb[r, 32 * j:32 * j + 32]).max())
                if rule == "floor":
                    m, e = np.frexp(b)                 # exact: b = m * 2^e, m in [0.5, 1)
                    X = (e - 1) - emax if b > 0 else -127
                else:
                    X = next(X for X in range(-200, 200) if b <= maxv * 2.0 ** X) if b > 0 else -127
                X = min(max(X, -127), 127)
                assert int(sf[oracle.sf_offset(r, j, 8)]) == X + 127, (rule, r, j, b)


@pytest.mark.parametrize("elem", ["e4m3", "e5m2"])
def test_mxfp8_ceil_rule_never_saturates_and_matches_torch_cast(elem):
    # Under the ceil rule every |x| <= max * 2^X, so no element clips and each
    # code is exactly torch's round-to-nearest-even cast of x * 2^-X.
    maxv = 448.0 if elem == "e4m3" else 57344.0
    tdt = torch.float8_e4m3fn if elem == "e4m3" else torch.float8_e5m2
    x = workloads.normal(128, 512, seed=29)
    x[9, 64:96] *= 1.75 / x[9, 64:96].float().abs().max()     # a block whose max is exactly 1.75 * 2^e
    codes, sf = oracle.mxfp8_quantize(bits(x), elem=elem, rule="ceil")
    xb = x.float().numpy()
    X = np.array([[int(sf[oracle.sf_offset(r, j, 16)]) - 127 for j in range(16)] for r in range(128)])
    Xe = np.repeat(X, 32, axis=1).astype(np.float64)
    assert np.all(np.abs(xb) <= maxv * np.exp2(Xe))
    scaled = torch.from_numpy((xb * np.exp2(-Xe)).astype(np.float32))   # exact: power-of-two scaling
    want = scaled.to(tdt).view(torch.uint8).numpy()
    assert np.array_equal(codes, want)
    codes_f, _ = oracle.mxfp8_quantize(bits(x), elem=elem, rule="floor")
    top = 0x7E if elem == "e4m3" else 0x7B
    assert ((codes_f & 0x7F) == top).sum() > ((codes & 0x7F) == top).sum()   # the floor rule clips some


@pytest.mark.parametrize("elem,rule", [("e5m2", "floor"), ("e5m2", "ceil"), ("e4m3", "ceil")])
@pytest.mark.parametrize("k", [-3, 5])
def test_mxfp8_variants_power_of_two_equivariance(elem, rule, k):
    x = workloads.normal(128, 256, seed=31)
    c0, s0 = oracle.mxfp8_quantize(bits(x), elem=elem, rule=rule)
    c1, s1 = oracle.mxfp8_quantize(bits((x.float() * 2.0 ** k).to(torch.bfloat16)), elem=elem, rule=rule)
    assert np.array_equal(c0, c1)
    nz = s0 != 0
    assert np.array_equal(s1[nz].astype(int), s0[nz].astype(int) + k)


def test_mxfp8_e5m2_dequantize_matches_library_decode():
    x = workloads.normal(128, 256, seed=37)
    codes, sf = oracle.mxfp8_quantize(bits(x), elem="e5m2")
    got = oracle.mxfp8_dequantize(codes, sf, 128, 256, elem="e5m2")
    vals = torch.from_numpy(codes).view(torch.float8_e5m2).double().numpy()
    scale = np.array([[torch.tensor([sf[oracle.sf_offset(r, k // 32, 8)]], dtype=torch.uint8)
                       .view(torch.float8_e8m0fnu).double().item() for k in range(256)] for r in range(128)])
    assert np.array_equal(got, vals * scale)


@pytest.mark.parametrize("M", [1, 100, 129])
def test_ragged_rows_equal_the_zero_padded_tensor(M):
    # A ragged row count quantizes its rows exactly as the zero-padded tensor
    # does (zero rows change neither amax nor any other row), and the scale
    # rows past M are zero.
    K = 256
    x = workloads.normal(M, K, seed=41 + M)
    Mp = (M + 127) // 128 * 128
    xp = torch.zeros(Mp, K, dtype=torch.bfloat16)
    xp[:M] = x
    c, s, g = oracle.nvfp4_quantize(bits(x))
    cp, sp, gp = oracle.nvfp4_quantize(bits(xp))
    assert g == gp and np.array_equal(c, cp[:M]) and np.array_equal(s, sp)
    for elem, rule in (("e4m3", "floor"), ("e5m2", "ceil")):
        c8, s8 = oracle.mxfp8_quantize(bits(x), elem=elem, rule=rule)
        c8p, s8p = oracle.mxfp8_quantize(bits(xp), elem=elem, rule=rule)
        assert np.array_equal(c8, c8p[:M])
        # padded rows: zero blocks give scale byte 0 (X = -127), the same as the zero padding
        assert np.array_equal(s8, s8p)
    nblk = K // 16
    assert all(s[oracle.sf_offset(r, j, nblk)] == 0 for r in range(M, Mp) for j in range(nblk))


# --------------------------------------------------------------------------
# Epilogue activation: binary64 -> BF16 rounding and GELU
# --------------------------------------------------------------------------

def _bf16_round_exact(v):
    """Independent reference: round a binary64 value to BF16 with exact
    rational arithmetic (nearest, ties to the even significand)."""
    from fractions import Fraction
    import math
    if v == 0:
        return 0x8000 if math.copysign(1.0, v) < 0 else 0
    sign = 0x8000 if v < 0 else 0
    a = Fraction(abs(v))
    e = math.floor(math.log2(abs(v)))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = Fraction(2) ** (max(e, -126) - 7)          # spacing of BF16 values here
    n = a / q
    fl = n.numerator // n.denominator
    rem = n - fl
    r = fl + (1 if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2) else 0)
    val = r * q
    if val >= Fraction(2) ** 128:
        return sign | 0x7F80
    f32 = np.float32(float(val))
    return sign | (int(np.array([f32]).view(np.uint32)[0]) >> 16) & 0x7FFF


def test_double_to_bf16_matches_exact_rounding_and_torch():
    # ties, values just off ties (where rounding through binary32 first would
    # give the wrong answer), subnormals, overflow
    cases = [1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -40, 1.0 + 2 ** -8 - 2 ** -40,
             -(1.0 + 2 ** -8 + 2 ** -40), 2.0 ** -133, 1.5 * 2.0 ** -133, 2.0 ** -134, 0.75 * 2.0 ** -133,
             2.0 ** -126 * 1.00390625, 3.3895313892515355e38, 3.4e38, 1e300, -0.0]
    for v in cases:
        assert oracle.double_to_bf16(v) == _bf16_round_exact(v), v
    # 1 + 2^-8 + 2^-40 is above the tie: rounds up, although binary32 rounding
    # first would land on the tie and then round to even (down)
    assert oracle.double_to_bf16(1.0 + 2 ** -8 + 2 ** -40) == 0x3F81
    rng = np.random.default_rng(43)
    vals = rng.standard_normal(5000) * np.exp2(rng.integers(-140, 120, 5000))
    for v in vals[:400]:
        assert oracle.double_to_bf16(float(v)) == _bf16_round_exact(float(v)), v
    # values exactly representable in binary32: one rounding, as torch's cast
    f32 = vals.astype(np.float32)
    want = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.double_to_bf16(float(v)) for v in f32], dtype=np.uint16)
    assert np.array_equal(got, want)


def _bf16_round_fraction(a, negative):
    """Nearest BF16 (ties to even) to the exact non-negative rational a."""
    from fractions import Fraction
    import math
    sign = 0x8000 if negative else 0
    if a == 0:
        return sign
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = Fraction(2) ** (max(e, -126) - 7)
    n = a / q
    fl = n.numerator // n.denominator
    rem = n - fl
    # the reference values are transcendental and carry about 300 bits: the
    # nearest one to a tie (a subnormal x, GELU(x) = x/2 + ~x^2 / sqrt(2 pi))
    # is about 2^-133 of a quantum away from it, far above their error
    assert abs(rem - Fraction(1, 2)) > Fraction(1, 2 ** 200)
    r = fl + (1 if rem > Fraction(1, 2) else 0)
    val = r * q
    if val >= Fraction(2) ** 128:
        return sign | 0x7F80
    f32 = np.float32(float(val))
    return sign | (int(np.array([f32]).view(np.uint32)[0]) >> 16) & 0x7FFF


def test_gelu_bf16_exhaustive_against_mpmath():
    """Every BF16 input: the oracle's GELU equals x * Phi(x) evaluated with
    90 significant digits (mpmath, independent of the C library's erfc) and
    rounded once to BF16 in exact rational arithmetic."""
    import mpmath
    from fractions import Fraction
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.gelu_bf16(bits)
    xs = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    mpmath.mp.dps = 90
    half_sqrt2 = mpmath.sqrt(2) / 2
    tiny = mpmath.mpf(2) ** -135
    for i in range(65536):
        x = float(xs[i])
        if np.isnan(x):
            assert (int(got[i]) & 0x7FFF) > 0x7F80, hex(i)      # NaN in, NaN out
            continue
        if np.isinf(x):
            assert int(got[i]) == (0x7F80 if x > 0 else 0x8000), hex(i)   # GELU(+inf) = inf, GELU(-inf) -> -0
            continue
        if x == 0.0:
            assert int(got[i]) == i & 0x8000, hex(i)
            continue
        g = mpmath.mpf(x) / 2 * mpmath.erfc(-mpmath.mpf(x) * half_sqrt2)
        if abs(g) < tiny:
            # below half the smallest BF16 subnormal (2^-133): rounds to -0
            # (x < -13.5; the value's exponent can reach -10^77)
            assert int(got[i]) == 0x8000, (hex(i), x)
            continue
        sign, man, exp, _ = g._mpf_
        a = Fraction(man) * (Fraction(2) ** exp if exp >= 0 else Fraction(1, 2 ** -exp))
        assert int(got[i]) == _bf16_round_fraction(a, bool(sign)), (hex(i), x)
    # closed forms: GELU(1) = Phi(1) = 0.8413447... -> BF16 0.83984375 (0x3F57);
    # GELU(10) = 10 (Phi(10) = 1 - 7.6e-24); GELU(-10) = -7.62e-23, which the
    # form 0.5 x (1 + erf(x / sqrt 2)) loses to cancellation in binary64
    assert int(got[0x3F80]) == 0x3F57
    assert int(got[0x4120]) == 0x4120
    g_m10 = float(torch.tensor([int(got[0xC120])], dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float())
    assert -7.7e-23 < g_m10 < -7.5e-23


def test_array_forms_equal_the_pinned_scalars():
    rng = np.random.default_rng(44)
    vals = np.concatenate([rng.standard_normal(3000) * np.exp2(rng.integers(-140, 120, 3000)),
                           [0.0, -0.0, np.inf, -np.inf, 1.0 + 2 ** -8, 1.0 + 2 ** -8 + 2 ** -40, 2.0 ** -134]])
    want = np.array([oracle.double_to_bf16(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(oracle.double_to_bf16_array(vals), want)
    assert np.array_equal(oracle.double_to_bf16_array(vals[:3003].reshape(-1, 7)), want[:3003].reshape(-1, 7))
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    assert np.array_equal(oracle.gelu_bf16_array(bits), oracle.gelu_bf16(bits))


def _bits_of(values):
    return torch.tensor(values, dtype=torch.float64).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_linear_gelu_mxfp8_closed_forms():
    """K = 32 with B the identity, so Y = A row by row (exact), then:
    row 0, values >= 4:     GELU is the identity on them, so the codes are
                            those of MXFP8(Y): block max 35 -> X = 5 - 8,
                            scale byte 124, code of v is E4M3(8 v);
    row 1, values <= -16:   GELU gives -0 everywhere: codes 0x80, scale 0
                            (a zero block takes X = -127);
    row 2, +-1 and 0:       GELU(1) = 0.8413 -> BF16 0x3F57 (0.83984375),
                            GELU(-1) = -0.1587 -> BF16 0xBE22 (-0.158203125);
                            block max 0.83984375 -> X = -1 - 8, codes of
                            0.83984375 * 512 = 430 -> 416 (spacing 32 in
                            [256, 512): 0x7D) and of -0.158203125 * 512 = -81
                            -> -80 (spacing 8 in [64, 128): 0xEA), 0 -> 0."""
    K = 32
    B = np.eye(K)
    row0 = np.arange(4, 36, dtype=np.float64)
    row1 = -np.arange(16, 48, dtype=np.float64)
    row2 = np.array([1.0, -1.0, 0.0, 1.0] * 8)
    A = np.stack([row0, row1, row2])
    codes, sf, D, G, Y = oracle.linear_gelu_mxfp8(A, B)
    assert np.array_equal(Y, A)
    assert np.array_equal(D, _bits_of(A))
    assert np.array_equal(G[0], D[0])
    assert np.all(G[1] == 0x8000)
    assert list(G[2][:4]) == [0x3F57, 0xBE22, 0x0000, 0x3F57]
    sfm = np.array([[sf[oracle.sf_offset(r, 0, 1)]] for r in range(3)])
    assert list(sfm[:, 0]) == [124, 0, 118]
    assert all(int(codes[0][i]) == oracle.e4m3_encode(8.0 * row0[i]) for i in range(K))
    assert int(codes[0][0]) == 0x60                          # 4 * 8 = 32 = 2^5
    assert np.all(codes[1] == 0x80)
    assert list(codes[2][:4]) == [0x7D, 0xEA, 0x00, 0x7D]
    # rows past the third, up to 128, are zero padding in the scale tile
    assert np.all(np.array([sf[oracle.sf_offset(r, 0, 1)] for r in range(3, 128)]) == 0)
