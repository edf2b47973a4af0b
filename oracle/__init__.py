"""CPU oracle for the microscaling-quantized linear layer (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
reference leg of ``bench.py`` may import this package.  The product path (the
CUDA library and its binding) never touches it.

This module is a thin ctypes wrapper over ``nvq_oracle.c``; every arithmetic
step lives in that C file.  Arrays are numpy: BF16 tensors travel as their
raw ``uint16`` bit patterns.
"""
import ctypes
import numpy as np

from . import build as _build

_lib = None

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64

NVFP4_BLOCK = 16
MXFP8_BLOCK = 32


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_e2m1_value.restype = ctypes.c_double
        L.oracle_e2m1_value.argtypes = [ctypes.c_int]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e4m3_value.argtypes = [ctypes.c_int]
        L.oracle_e8m0_value.restype = ctypes.c_double
        L.oracle_e8m0_value.argtypes = [ctypes.c_int]
        L.oracle_e2m1_encode.restype = ctypes.c_int
        L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_int
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode_array.restype = None
        L.oracle_e4m3_encode_array.argtypes = [_f32p, _i64, _u8p]
        L.oracle_take_nan_flag.restype = ctypes.c_int
        L.oracle_sf_bytes.restype = _i64
        L.oracle_sf_bytes.argtypes = [_i64, _i64]
        L.oracle_sf_offset.restype = _i64
        L.oracle_sf_offset.argtypes = [_i64, _i64, _i64]
        L.oracle_amax.restype = ctypes.c_float
        L.oracle_amax.argtypes = [_u16p, _i64, _i64, _i64]
        L.oracle_nvfp4_quantize.restype = None
        L.oracle_nvfp4_quantize.argtypes = [_u16p, _i64, _i64, _i64, _f32p, _u8p, _u8p, _f32p]
        L.oracle_nvfp4_dequantize.restype = None
        L.oracle_nvfp4_dequantize.argtypes = [_u8p, _u8p, ctypes.c_float, _i64, _i64, _f64p]
        L.oracle_mxfp8_quantize.restype = None
        L.oracle_mxfp8_quantize.argtypes = [_u16p, _i64, _i64, _i64, _u8p, _u8p]
        L.oracle_mxfp8_dequantize.restype = None
        L.oracle_mxfp8_dequantize.argtypes = [_u8p, _u8p, _i64, _i64, _f64p]
        L.oracle_mxfp8_quantize_ex.restype = None
        L.oracle_mxfp8_quantize_ex.argtypes = [_u16p, _i64, _i64, _i64, ctypes.c_int, ctypes.c_int, _u8p, _u8p]
        L.oracle_mxfp8_dequantize_ex.restype = None
        L.oracle_mxfp8_dequantize_ex.argtypes = [_u8p, _u8p, _i64, _i64, ctypes.c_int, _f64p]
        L.oracle_double_to_bf16.restype = ctypes.c_uint16
        L.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        L.oracle_gelu_bf16.restype = ctypes.c_uint16
        L.oracle_gelu_bf16.argtypes = [ctypes.c_uint16]
        L.oracle_double_to_bf16_array.restype = None
        L.oracle_double_to_bf16_array.argtypes = [_f64p, _i64, _u16p]
        L.oracle_gelu_bf16_array.restype = None
        L.oracle_gelu_bf16_array.argtypes = [_u16p, _i64, _u16p]
        L.oracle_e5m2_value.restype = ctypes.c_double
        L.oracle_e5m2_value.argtypes = [ctypes.c_int]
        L.oracle_e5m2_encode.restype = ctypes.c_int
        L.oracle_e5m2_encode.argtypes = [ctypes.c_float]
        L.oracle_gemm_rows.restype = None
        L.oracle_gemm_rows.argtypes = [_f64p, _f64p, _i64, _i64, _i64p, _i64, _u16p, _f64p]
        L.oracle_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a, t):
    return a.ctypes.data_as(t)


def _bf16_bits(x):
    """Accept a numpy uint16 array of BF16 bit patterns or a torch bf16 tensor."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        x = x.contiguous().view(dtype=__import__("torch").int16).numpy().view(np.uint16)
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16 and x.ndim == 2
    return x


# --- element formats -------------------------------------------------------

def e2m1_value(code):
    return lib().oracle_e2m1_value(int(code))


def e4m3_value(code):
    return lib().oracle_e4m3_value(int(code))


def e5m2_value(code):
    return lib().oracle_e5m2_value(int(code))


def e5m2_encode(v):
    return lib().oracle_e5m2_encode(float(np.float32(v)))


def e8m0_value(code):
    return lib().oracle_e8m0_value(int(code))


def e2m1_encode(v):
    return lib().oracle_e2m1_encode(float(np.float32(v)))


def e4m3_encode(v):
    return lib().oracle_e4m3_encode(float(np.float32(v)))


def e4m3_encode_array(v):
    """Elementwise e4m3_encode of an array of FP32 values (same shape, uint8 codes)."""
    a = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_array(_ptr(a, _f32p), a.size, _ptr(out, _u8p))
    return out


def take_nan_flag():
    return bool(lib().oracle_take_nan_flag())


# --- scale layout ----------------------------------------------------------

def sf_bytes(rows, cols):
    return int(lib().oracle_sf_bytes(rows, cols))


def sf_offset(r, c, cols):
    return int(lib().oracle_sf_offset(r, c, cols))


# --- quantization ------------------------------------------------------------

def amax(x_bits, ldx=None):
    x = _bf16_bits(x_bits)
    M, K = x.shape
    return float(lib().oracle_amax(_ptr(x, _u16p), M, K, ldx or K))


def nvfp4_quantize(x_bits, calib_amax=None):
    """Returns (codes u8 [M, K/2], sf u8 [sf_bytes(M, K/16)], g_dec float32)."""
    x = _bf16_bits(x_bits)
    M, K = x.shape
    assert K % NVFP4_BLOCK == 0
    codes = np.zeros((M, K // 2), dtype=np.uint8)
    sf = np.zeros(sf_bytes(M, K // NVFP4_BLOCK), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    ca = None
    if calib_amax is not None:
        ca_arr = np.array([calib_amax], dtype=np.float32)
        ca = _ptr(ca_arr, _f32p)
    lib().oracle_nvfp4_quantize(_ptr(x, _u16p), M, K, K, ca, _ptr(codes, _u8p), _ptr(sf, _u8p), _ptr(g, _f32p))
    return codes, sf, np.float32(g[0])


def nvfp4_dequantize(codes, sf, g_dec, rows, K):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    out = np.empty((rows, K), dtype=np.float64)
    lib().oracle_nvfp4_dequantize(_ptr(codes, _u8p), _ptr(sf, _u8p), float(g_dec), rows, K, _ptr(out, _f64p))
    return out


def double_to_bf16(v):
    """binary64 -> BF16 bit pattern, one round-to-nearest-even."""
    return int(lib().oracle_double_to_bf16(float(v)))


def gelu_bf16(bits_arr):
    """GELU (exact erf, binary64) of BF16 bit patterns, rounded once to BF16."""
    a = np.ascontiguousarray(bits_arr, dtype=np.uint16)
    f = lib().oracle_gelu_bf16
    return np.vectorize(lambda b: f(int(b)), otypes=[np.uint16])(a)


def double_to_bf16_array(v):
    """Elementwise double_to_bf16 of a binary64 array (same shape, uint16 bits)."""
    a = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().oracle_double_to_bf16_array(_ptr(a, _f64p), a.size, _ptr(out, _u16p))
    return out


def gelu_bf16_array(bits_arr):
    """Elementwise gelu_bf16 of BF16 bit patterns (same shape, uint16 bits)."""
    a = np.ascontiguousarray(bits_arr, dtype=np.uint16)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().oracle_gelu_bf16_array(_ptr(a, _u16p), a.size, _ptr(out, _u16p))
    return out


ELEMS = {"e4m3": 0, "e5m2": 1}
RULES = {"floor": 0, "ceil": 1}


def mxfp8_quantize(x_bits, elem="e4m3", rule="floor"):
    """Returns (codes u8 [M, K], sf u8 [sf_bytes(M, K/32)]).
    elem: "e4m3" or "e5m2" elements; rule: "floor" (OCP) or "ceil" block exponent."""
    x = _bf16_bits(x_bits)
    M, K = x.shape
    assert K % MXFP8_BLOCK == 0
    codes = np.zeros((M, K), dtype=np.uint8)
    sf = np.zeros(sf_bytes(M, K // MXFP8_BLOCK), dtype=np.uint8)
    lib().oracle_mxfp8_quantize_ex(_ptr(x, _u16p), M, K, K, ELEMS[elem], RULES[rule], _ptr(codes, _u8p),
                                   _ptr(sf, _u8p))
    return codes, sf


def mxfp8_dequantize(codes, sf, rows, K, elem="e4m3"):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    out = np.empty((rows, K), dtype=np.float64)
    lib().oracle_mxfp8_dequantize_ex(_ptr(codes, _u8p), _ptr(sf, _u8p), rows, K, ELEMS[elem], _ptr(out, _f64p))
    return out


# --- GEMM ------------------------------------------------------------------------

def gemm_rows(A_hat, B_hat, rows=None, bias_bits=None):
    """out[i, n] = sum_k A_hat[rows[i], k] * B_hat[n, k] (+ bias[n]), binary64."""
    A = np.ascontiguousarray(A_hat, dtype=np.float64)
    B = np.ascontiguousarray(B_hat, dtype=np.float64)
    N, K = B.shape
    assert A.shape[1] == K
    if rows is None:
        rows = np.arange(A.shape[0], dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty((rows.size, N), dtype=np.float64)
    bp = None
    if bias_bits is not None:
        bias = np.ascontiguousarray(bias_bits, dtype=np.uint16).reshape(-1)
        assert bias.size == N
        bp = _ptr(bias, _u16p)
    lib().oracle_gemm_rows(_ptr(A, _f64p), _ptr(B, _f64p), N, K, _ptr(rows, _i64p), rows.size, bp, _ptr(out, _f64p))
    return out


def linear_gelu_mxfp8(A_hat, B_hat, rows=None, bias_bits=None):
    """The first linear of a feed-forward block followed by the next layer's
    activation quantization, in the order the definitions give:
      Y = A_hat[rows] . B_hat^T (+ bias), binary64        (gemm_rows)
      D = Y rounded once to BF16                            (double_to_bf16)
      G = GELU(D) = D * Phi(D), rounded once to BF16        (gelu_bf16)
      codes, sf = MXFP8 of G (E4M3 elements, floor rule)    (mxfp8_quantize)
    Returns (codes u8 [R, N], sf u8 (tile order over R rows), D bits, G bits, Y)
    with R = len(rows)."""
    Y = gemm_rows(A_hat, B_hat, rows=rows, bias_bits=bias_bits)
    D = double_to_bf16_array(Y)
    G = gelu_bf16_array(D)
    codes, sf = mxfp8_quantize(G)
    return codes, sf, D, G, Y


def num_threads():
    return int(lib().oracle_num_threads())


# --- acceptance rule --------------------------------------------------------------

GEMM_TOL = 2e-3


def bf16_rounding_interval(D):
    """[lo, hi]: the real values that round to nearest (ties to even, taken
    inclusively) to the BF16 value D, elementwise.  D must hold BF16 values
    (the output's own format).  Half the spacing to the next BF16 magnitude
    lies above |D| and half the spacing to the previous one below it (the
    two differ at a power of two); +-0 covers half the smallest subnormal on
    each side.  Non-finite D gives an empty interval (lo = +inf, hi = -inf)."""
    D = np.asarray(D, dtype=np.float64)
    f = D.astype(np.float32)
    bits = f.view(np.uint32)
    assert np.all((f.astype(np.float64) == D) | np.isnan(D)) and np.all((bits & 0xFFFF) == 0), \
        "D must hold BF16 values"
    m = (bits >> 16) & 0x7FFF
    val = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    mag = val(m)
    finite = m < 0x7F80
    prev = val(np.where(m > 0, m - 1, 0))
    nxt = val(np.where(m + 1 < 0x7F80, m + 1, 0))
    up = np.where(m + 1 < 0x7F80, nxt - mag, mag - prev)     # spacing above |D| (the top binade's, at the largest)
    down_half = np.where(m > 0, (mag - prev) / 2, 2.0 ** -134)
    neg = (bits >> 31) == 1
    with np.errstate(invalid="ignore"):
        lo = np.where(neg, -(mag + up / 2), mag - down_half)
        hi = np.where(neg, -(mag - down_half), mag + up / 2)
    return np.where(finite, lo, np.inf), np.where(finite, hi, -np.inf)


def gemm_row_errors(D, Y):
    """The GEMM acceptance rule: the output is judged before its BF16
    rounding, which the tests cannot observe, so a BF16 output D[row, n] is
    correct when some value that rounds to it lies near Y[row, n].  Per row:
    max_n dist(Y[row, n], rounding interval of D[row, n]) / ||Y[row, :]||_2,
    with an all-zero reference row allowing only +-0 outputs (its error is 0
    or inf).  D = BF16 rounding of Y gives 0 on every row."""
    Y = np.asarray(Y, dtype=np.float64)
    lo, hi = bf16_rounding_interval(D)
    err = np.maximum(np.maximum(lo - Y, Y - hi), 0.0)
    err = np.where(np.isfinite(lo), err, np.inf).max(axis=1)
    nrm = np.linalg.norm(Y, axis=1)
    zero_row = np.where(err > 0, np.inf, 0.0)
    return np.where(nrm > 0, err / np.where(nrm > 0, nrm, 1.0), zero_row)
