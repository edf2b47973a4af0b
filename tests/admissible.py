"""Admissible outputs of the fused GELU + MXFP8 epilogue (test infrastructure).

The epilogue's codes and scales are a function of the linear's BF16 result D,
and D is known only to the GEMM's tolerance, which judges the result before
its BF16 rounding: the BF16 rounding of any value within tol * ||Y row||_2 of
the oracle's binary64 sum Y is a correct D (oracle.gemm_row_errors).  So several
outputs are correct, and check_admissible() accepts exactly those bytes that
some admissible D explains, element by element and block by block, with no
allowance for a count of mismatches.  Every value it compares comes from the
oracle (its BF16 rounding, its GELU, its E4M3 encoder)."""
import numpy as np

import oracle


def _bf16_val(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# GELU falls, then rises, with its minimum at x* = -0.7518 (between the BF16
# values -0.7539 and -0.75); every BF16 value in [-0.78, -0.72] is kept as a
# candidate for the smallest GELU of an interval that contains x*.
_NEAR_MIN = np.array([b for b in range(0xBF38, 0xBF49) if -0.78 <= _bf16_val(np.uint16(b)) <= -0.72],
                     dtype=np.uint16)
_E4M3_VALUES = np.array([np.nan if c & 0x7F == 0x7F else oracle.e4m3_value(c) for c in range(256)])


def admissible_gelu(Y, tol=oracle.GEMM_TOL):
    """For every element: the smallest and largest BF16 GELU(D) over the BF16
    values D that are the rounding of a value within tol * ||Y row||_2 of the
    binary64 sum Y (the GEMM's acceptance rule).  Rounding to nearest is
    monotone, so those D are the BF16 values from the rounding of Y - t to
    the rounding of Y + t.  GELU decreases below x* and increases above it,
    and rounding to BF16 keeps that order, so the largest value sits at an
    end of that range and the smallest at an end or at the BF16 neighbour of
    x*."""
    t = tol * np.linalg.norm(Y, axis=1, keepdims=True)
    a, b = oracle.double_to_bf16_array(Y - t), oracle.double_to_bf16_array(Y + t)
    va, vb = _bf16_val(a), _bf16_val(b)
    ga, gb = _bf16_val(oracle.gelu_bf16_array(a)), _bf16_val(oracle.gelu_bf16_array(b))
    gmin, gmax = np.minimum(ga, gb), np.maximum(ga, gb)
    for c, gc in zip(_bf16_val(_NEAR_MIN), _bf16_val(oracle.gelu_bf16_array(_NEAR_MIN))):
        gmin = np.where((va <= c) & (c <= vb), np.minimum(gmin, gc), gmin)
    return gmin, gmax


def _mx_exponent(m):
    """OCP floor rule: floor(log2 m) - 8 clamped to [-127, 127]; -127 for m = 0."""
    _, e = np.frexp(m)
    return np.clip(np.where(m > 0, e - 1 - 8, -127), -127, 127)


def check_admissible(codes, sf_bytes, Y, tol=oracle.GEMM_TOL):
    """No byte outside what some admissible D allows.  codes u8 [R, N] and
    sf_bytes u8 [R, N / 32] (logical order) are the kernel's outputs for the
    rows whose binary64 sums are Y [R, N].
      scales: the block max of |G| lies between max_i min|G_i| and
        max_i max|G_i|, so the E8M0 byte lies between the exponents of those;
      codes: under the byte the kernel chose, E4M3(G * 2^-X) is monotone in
        G, so each code lies between the codes of the smallest and the
        largest admissible G of its element."""
    R, N = Y.shape
    gmin, gmax = admissible_gelu(Y, tol)
    lo_abs = np.where((gmin <= 0) & (gmax >= 0), 0.0, np.minimum(np.abs(gmin), np.abs(gmax)))
    hi_abs = np.maximum(np.abs(gmin), np.abs(gmax))
    s_lo = _mx_exponent(lo_abs.reshape(R, N // 32, 32).max(axis=2)) + 127
    s_hi = _mx_exponent(hi_abs.reshape(R, N // 32, 32).max(axis=2)) + 127
    s = sf_bytes.astype(np.int64)
    bad = np.argwhere((s < s_lo) | (s > s_hi))
    assert bad.size == 0, "%d inadmissible scale bytes, first at %s: %d not in [%d, %d]" % (
        len(bad), bad[0], s[tuple(bad[0])], s_lo[tuple(bad[0])], s_hi[tuple(bad[0])])
    mult = np.exp2(-np.repeat(s - 127, 32, axis=1).astype(np.float64))
    c_lo = oracle.e4m3_encode_array(np.clip(gmin * mult, -1e6, 1e6).astype(np.float32))
    c_hi = oracle.e4m3_encode_array(np.clip(gmax * mult, -1e6, 1e6).astype(np.float32))
    v, v_lo, v_hi = _E4M3_VALUES[codes], _E4M3_VALUES[c_lo], _E4M3_VALUES[c_hi]
    bad = np.argwhere(~((v_lo <= v) & (v <= v_hi)))
    assert bad.size == 0, "%d inadmissible codes, first at %s: %02x not in [%02x, %02x]" % (
        len(bad), bad[0], codes[tuple(bad[0])], c_lo[tuple(bad[0])], c_hi[tuple(bad[0])])
    return int(np.count_nonzero(s_lo != s_hi)), int(np.count_nonzero(c_lo != c_hi))
