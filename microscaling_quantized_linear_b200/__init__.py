"""Python binding of ``libnvq.so``: the B200 microscaling-quantized linear layer.

Argument marshalling only.  Every step of quantization and of the GEMM runs
in the CUDA kernels behind the C ABI declared in ``include/nvq.h``; this
module turns torch tensors into device pointers and the current CUDA stream,
allocates output tensors with torch when the caller does not pass them, and
raises ``NvqError`` on a non-zero return code.  There is no fallback: if the
shared library is missing, importing this package fails.

Names follow the C ABI: ``nvfp4_quantize`` (and ``nvfp4_quantize_noalloc``),
``mxfp8_quantize``, ``quantize_weight``, ``block_scaled_linear``,
``block_scaled_linear_gelu_mxfp8``, ``nvfp4_linear_short_m``, plus the size
helpers, the status word and the test hooks.  ``QuantizedLinear`` sequences
them for a caller: weight quantized once, then per call the activation's
quantization and the GEMM (one launch for NVFP4 batches of at most 8 rows).

With NVQ_DEBUG=1 in the environment at import, the debug build
``libnvq_debug.so`` (bounds-checked kernels, see ``build.py``) is loaded
instead; ``DEBUG_BUILD`` says which one is in use.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_WANT_DEBUG = os.environ.get("NVQ_DEBUG", "") not in ("", "0")
LIB_PATH = os.path.join(_HERE, "libnvq_debug.so" if _WANT_DEBUG else "libnvq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "%s is not built (expected at %s); run "
        "`python microscaling_quantized_linear_b200/build.py%s` or __graft_entry__.build()"
        % (os.path.basename(LIB_PATH), LIB_PATH, " --debug" if _WANT_DEBUG else ""))

_lib = ctypes.CDLL(LIB_PATH)

NVFP4 = 0
MXFP8 = 1
MXFP8_E5M2 = 2
_FORMATS = {"nvfp4": NVFP4, "mxfp8": MXFP8, "mxfp8_e5m2": MXFP8_E5M2,
            NVFP4: NVFP4, MXFP8: MXFP8, MXFP8_E5M2: MXFP8_E5M2}
SCALE_FLOOR = 0
SCALE_CEIL = 1
_ELEMS = {"e4m3": MXFP8, "e5m2": MXFP8_E5M2}
_RULES = {"floor": SCALE_FLOOR, "ceil": SCALE_CEIL}

NVQ_STATUS_TIMEOUT = 1
NVQ_STATUS_NONFINITE = 2
NVQ_STATUS_WORKSPACE = 4
NVQ_STATUS_BOUNDS = 8

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t

_lib.nvq_codes_bytes.restype = _sz
_lib.nvq_codes_bytes.argtypes = [ctypes.c_int, _i64, _i64]
_lib.nvq_scale_bytes.restype = _sz
_lib.nvq_scale_bytes.argtypes = [ctypes.c_int, _i64, _i64]
_lib.nvq_workspace_bytes.restype = _sz
_lib.nvq_workspace_bytes.argtypes = []
_lib.nvfp4_quantize.restype = ctypes.c_int
_lib.nvfp4_quantize.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.mxfp8_quantize.restype = ctypes.c_int
_lib.mxfp8_quantize.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp, _vp]
_lib.mxfp8_quantize_ex.restype = ctypes.c_int
_lib.mxfp8_quantize_ex.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp, ctypes.c_int, ctypes.c_int, _vp]
_lib.quantize_weight.restype = ctypes.c_int
_lib.quantize_weight.argtypes = [ctypes.c_int, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp]
_lib.block_scaled_linear.restype = ctypes.c_int
_lib.block_scaled_linear.argtypes = [ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64,
                                     _i64, _i64, _i64, _vp]
_lib.nvq_device_status.restype = ctypes.c_int
_lib.nvq_device_status.argtypes = [_vp]
_lib.nvq_status_string.restype = ctypes.c_char_p
_lib.nvq_status_string.argtypes = [ctypes.c_int]
_lib.nvq_probe_convert.restype = ctypes.c_int
_lib.nvq_probe_convert.argtypes = [_vp, _i64, _vp, _vp, _vp]
_lib.nvfp4_quantize_noalloc.restype = ctypes.c_int
_lib.nvfp4_quantize_noalloc.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp]
_lib.block_scaled_linear_gelu_mxfp8.restype = ctypes.c_int
_lib.block_scaled_linear_gelu_mxfp8.argtypes = [ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                                _i64, _i64, _i64, _vp]
_lib.nvfp4_linear_short_m.restype = ctypes.c_int
_lib.nvfp4_linear_short_m.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp]
_lib.nvq_probe_gelu.restype = ctypes.c_int
_lib.nvq_probe_gelu.argtypes = [_vp, _i64, _vp, _vp]
_lib.nvq_probe_wait.restype = ctypes.c_int
_lib.nvq_probe_wait.argtypes = [ctypes.c_uint64, _vp, _vp]
_lib.nvq_gemm_plan.restype = ctypes.c_int
_lib.nvq_gemm_plan.argtypes = [ctypes.c_int, _i64, _i64, _i64, _vp, _vp, _vp]
_lib.nvq_debug_build.restype = ctypes.c_int
_lib.nvq_debug_build.argtypes = []
_lib.nvq_probe_bounds.restype = ctypes.c_int
_lib.nvq_probe_bounds.argtypes = [_vp]
_lib.nvq_set_wait_limit.restype = ctypes.c_int
_lib.nvq_set_wait_limit.argtypes = [ctypes.c_uint64]
_lib.nvq_wait_limit.restype = ctypes.c_uint64
_lib.nvq_wait_limit.argtypes = []
_lib.nvq_workspace_init.restype = ctypes.c_int
_lib.nvq_workspace_init.argtypes = [_vp, _vp]
_lib.nvq_gemm_plan_host.restype = ctypes.c_int
_lib.nvq_gemm_plan_host.argtypes = [ctypes.c_int, _i64, _i64, _i64, ctypes.c_int, _vp, ctypes.c_int, ctypes.c_int,
                                    _vp, _vp, _vp]

EXPORTED = ("nvq_codes_bytes", "nvq_scale_bytes", "nvq_workspace_bytes", "nvfp4_quantize",
            "mxfp8_quantize", "mxfp8_quantize_ex", "quantize_weight", "block_scaled_linear",
            "nvq_device_status", "nvq_status_string", "nvq_probe_convert", "nvfp4_quantize_noalloc",
            "block_scaled_linear_gelu_mxfp8", "nvq_probe_gelu", "nvq_probe_wait", "nvq_gemm_plan",
            "nvq_gemm_plan_host", "nvq_set_wait_limit", "nvq_workspace_init", "nvq_debug_build",
            "nvq_probe_bounds", "nvfp4_linear_short_m", "nvq_wait_limit")

DEBUG_BUILD = bool(_lib.nvq_debug_build())

NOALLOC_MAX_PARTIALS = 1024


class NvqError(RuntimeError):
    def __init__(self, code, what):
        self.code = code
        super().__init__("%s failed: %s (%d)" % (what, status_string(code), code))


def status_string(code):
    return _lib.nvq_status_string(int(code)).decode()


def _check(rc, what):
    if rc != 0:
        raise NvqError(rc, what)


def _fmt(f):
    try:
        return _FORMATS[f]
    except KeyError:
        raise ValueError("unknown format %r" % (f,)) from None


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _buf(t, dtype, nbytes, name):
    """A device buffer that the call reads or writes as nbytes contiguous
    bytes: checked before the library sees its pointer, since the C ABI
    cannot check the size of what a pointer points to."""
    if t.dtype != dtype:
        raise ValueError("%s: expected %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s: expected a contiguous tensor" % name)
    if t.numel() * t.element_size() < nbytes:
        raise ValueError("%s: %d bytes, the call needs %d" % (name, t.numel() * t.element_size(), nbytes))
    return t


def _mat(t, dtype, rows, cols, name):
    """A row-major [rows, cols] matrix with unit column stride (any row pitch)."""
    if t.dtype != dtype:
        raise ValueError("%s: expected %s, got %s" % (name, dtype, t.dtype))
    if t.dim() != 2 or tuple(t.shape) != (rows, cols) or t.stride(1) != 1:
        raise ValueError("%s: expected a [%d, %d] matrix with unit column stride, got shape %s strides %s"
                         % (name, rows, cols, tuple(t.shape), tuple(t.stride())))
    return t


def _cuda(**tensors):
    """Every tensor given (None skipped) lives on a CUDA device (checked after
    the dtypes and sizes)."""
    for name, t in tensors.items():
        if t is not None and not t.is_cuda:
            raise ValueError("%s: expected a CUDA tensor" % name)


def _pitch(t):
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit stride in the last dimension")
    return t.stride(0)


# --------------------------------------------------------------------------- sizes

def codes_bytes(fmt, rows, K):
    return int(_lib.nvq_codes_bytes(_fmt(fmt), rows, K))


def scale_bytes(fmt, rows, K):
    return int(_lib.nvq_scale_bytes(_fmt(fmt), rows, K))


def workspace_bytes():
    return int(_lib.nvq_workspace_bytes())


def new_workspace(device="cuda"):
    """A workspace for nvfp4_quantize / quantize_weight, zero-filled as its
    first use requires (every call then leaves it ready for the next)."""
    return torch.zeros(workspace_bytes(), dtype=torch.uint8, device=device)


def workspace_init(workspace, stream=None):
    """Zero-fill a workspace through the library (nvq_workspace_init)."""
    _check(_lib.nvq_workspace_init(_ptr(workspace), _stream(stream, workspace.device)), "nvq_workspace_init")


# --------------------------------------------------------------------------- quantizers

def _nvfp4_args(x, codes, scales, global_scale):
    M, K = x.shape
    _mat(x, torch.bfloat16, M, K, "x")
    _buf(codes, torch.uint8, codes_bytes(NVFP4, M, K), "codes")
    _buf(scales, torch.uint8, scale_bytes(NVFP4, M, K), "scales")
    _buf(global_scale, torch.float32, 4, "global_scale")


def nvfp4_quantize(x, codes=None, scales=None, global_scale=None, calib_amax=None, workspace=None,
                   stream=None):
    """BF16 [M, K] -> (codes u8 [M, K/2], scales u8 (tile order), global_scale f32 [1])."""
    M, K = x.shape
    dev = x.device
    codes = codes if codes is not None else torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    scales = scales if scales is not None else torch.empty(scale_bytes(NVFP4, M, K), dtype=torch.uint8, device=dev)
    global_scale = global_scale if global_scale is not None else torch.empty(1, dtype=torch.float32, device=dev)
    if workspace is None and calib_amax is None:
        workspace = new_workspace(dev)
    _nvfp4_args(x, codes, scales, global_scale)
    if calib_amax is not None:
        _buf(calib_amax, torch.float32, 4, "calib_amax")
    if workspace is not None:
        _buf(workspace, torch.uint8, workspace_bytes(), "workspace")
    _cuda(x=x, codes=codes, scales=scales, global_scale=global_scale, calib_amax=calib_amax, workspace=workspace)
    _check(_lib.nvfp4_quantize(_ptr(x), M, K, _pitch(x), _ptr(codes), _ptr(scales), _ptr(global_scale),
                               _ptr(calib_amax), _ptr(workspace), _stream(stream, dev)), "nvfp4_quantize")
    return codes, scales, global_scale


def nvfp4_quantize_noalloc(x, codes, scales, global_scale, stream=None):
    """nvfp4_quantize (dynamic amax) through the entry point that needs no
    workspace and allocates nothing: its scratch is a static array inside the
    library.  The outputs must be given (this call allocates nothing)."""
    M, K = x.shape
    _nvfp4_args(x, codes, scales, global_scale)
    _cuda(x=x, codes=codes, scales=scales, global_scale=global_scale)
    _check(_lib.nvfp4_quantize_noalloc(_ptr(x), M, K, _pitch(x), _ptr(codes), _ptr(scales), _ptr(global_scale),
                                       _stream(stream, x.device)), "nvfp4_quantize_noalloc")
    return codes, scales, global_scale


def mxfp8_quantize(x, codes=None, scales=None, stream=None, elem="e4m3", rule="floor"):
    """BF16 [M, K] -> (codes u8 [M, K] (E4M3 or E5M2), scales u8 (E8M0, tile order)).
    elem "e4m3" | "e5m2"; rule "floor" (OCP) | "ceil" (no element saturates)."""
    M, K = x.shape
    dev = x.device
    codes = codes if codes is not None else torch.empty((M, K), dtype=torch.uint8, device=dev)
    scales = scales if scales is not None else torch.empty(scale_bytes(MXFP8, M, K), dtype=torch.uint8, device=dev)
    _mat(x, torch.bfloat16, M, K, "x")
    _buf(codes, torch.uint8, codes_bytes(MXFP8, M, K), "codes")
    _buf(scales, torch.uint8, scale_bytes(MXFP8, M, K), "scales")
    _cuda(x=x, codes=codes, scales=scales)
    if elem == "e4m3" and rule == "floor":
        rc = _lib.mxfp8_quantize(_ptr(x), M, K, _pitch(x), _ptr(codes), _ptr(scales), _stream(stream, dev))
    else:
        if elem not in _ELEMS or rule not in _RULES:
            raise ValueError("unknown element type %r or rule %r" % (elem, rule))
        rc = _lib.mxfp8_quantize_ex(_ptr(x), M, K, _pitch(x), _ptr(codes), _ptr(scales), _ELEMS[elem],
                                    _RULES[rule], _stream(stream, dev))
    _check(rc, "mxfp8_quantize")
    return codes, scales


def quantize_weight(fmt, w, codes=None, scales=None, global_scale=None, workspace=None, stream=None):
    """Offline weight quantization; returns (codes, scales, global_scale or None)."""
    f = _fmt(fmt)
    N, K = w.shape
    dev = w.device
    cols = K // 2 if f == NVFP4 else K     # MXFP8 (either element type): one byte per value
    codes = codes if codes is not None else torch.empty((N, cols), dtype=torch.uint8, device=dev)
    scales = scales if scales is not None else torch.empty(scale_bytes(f, N, K), dtype=torch.uint8, device=dev)
    if f == NVFP4:
        global_scale = global_scale if global_scale is not None else torch.empty(1, dtype=torch.float32, device=dev)
        workspace = workspace if workspace is not None else new_workspace(dev)
        _buf(global_scale, torch.float32, 4, "global_scale")
        _buf(workspace, torch.uint8, workspace_bytes(), "workspace")
    _mat(w, torch.bfloat16, N, K, "w")
    _buf(codes, torch.uint8, codes_bytes(f, N, K), "codes")
    _buf(scales, torch.uint8, scale_bytes(f, N, K), "scales")
    _cuda(w=w, codes=codes, scales=scales, global_scale=global_scale, workspace=workspace)
    _check(_lib.quantize_weight(f, _ptr(w), N, K, _pitch(w), _ptr(codes), _ptr(scales), _ptr(global_scale),
                                _ptr(workspace), _stream(stream, dev)), "quantize_weight")
    return codes, scales, global_scale


# --------------------------------------------------------------------------- GEMM

def _gemm_args(f, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias, M, N, K):
    _buf(a_codes, torch.uint8, codes_bytes(f, M, K), "a_codes")
    _buf(a_scales, torch.uint8, scale_bytes(f, M, K), "a_scales")
    _buf(b_codes, torch.uint8, codes_bytes(f, N, K), "b_codes")
    _buf(b_scales, torch.uint8, scale_bytes(f, N, K), "b_scales")
    if f == NVFP4:
        if a_global is None or b_global is None:
            raise ValueError("NVFP4 operands need their global scales")
        _buf(a_global, torch.float32, 4, "a_global")
        _buf(b_global, torch.float32, 4, "b_global")
    if bias is not None:
        _buf(bias, torch.bfloat16, 2 * N, "bias")


def _gemm_cuda(a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias, **outs):
    _cuda(a_codes=a_codes, a_scales=a_scales, a_global=a_global, b_codes=b_codes, b_scales=b_scales,
          b_global=b_global, bias=bias, **outs)


def block_scaled_linear(fmt, a_codes, a_scales, a_global, b_codes, b_scales, b_global, M, N, K,
                        bias=None, out=None, stream=None):
    """D = bf16(alpha * A . B^T + bias) on the block-scaled tensor cores; returns out [M, N]."""
    f = _fmt(fmt)
    dev = a_codes.device
    out = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    _gemm_args(f, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias, M, N, K)
    _mat(out, torch.bfloat16, M, N, "out")
    _gemm_cuda(a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias, out=out)
    _check(_lib.block_scaled_linear(f, _ptr(a_codes), _ptr(a_scales), _ptr(a_global), _ptr(b_codes),
                                    _ptr(b_scales), _ptr(b_global), _ptr(bias), _ptr(out), _pitch(out),
                                    M, N, K, _stream(stream, dev)), "block_scaled_linear")
    return out


def gemm_plan(fmt, M, N, K):
    """The kernel block_scaled_linear launches for this shape on the current
    device: (tile_m, tile_n, k_split); tile_m 256 is a CTA pair, k_split > 1
    a cluster of CTAs splitting K.  Host-only."""
    tm, tn, ks = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(_lib.nvq_gemm_plan(_fmt(fmt), M, N, K, ctypes.byref(tm), ctypes.byref(tn), ctypes.byref(ks)),
           "nvq_gemm_plan")
    return tm.value, tn.value, ks.value


def gemm_plan_host(fmt, M, N, K, num_sms, max_clusters, use_pairs=True, use_splitk=True):
    """gemm_plan for stated device facts: num_sms and max_clusters, a mapping
    {(tile_n, k_split): clusters the device holds at once} (missing entries
    count as 0).  Host-only; needs no GPU."""
    table = (ctypes.c_int * 27)()
    for (tn, ks), n in max_clusters.items():
        table[(tn // 64 - 2) * 9 + ks] = int(n)
    tm, tn_, ks_ = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(_lib.nvq_gemm_plan_host(_fmt(fmt), M, N, K, int(num_sms), table, int(bool(use_pairs)),
                                   int(bool(use_splitk)), ctypes.byref(tm), ctypes.byref(tn_), ctypes.byref(ks_)),
           "nvq_gemm_plan_host")
    return tm.value, tn_.value, ks_.value


def block_scaled_linear_gelu_mxfp8(fmt, a_codes, a_scales, a_global, b_codes, b_scales, b_global, M, N, K,
                                   bias=None, y_codes=None, y_scales=None, stream=None):
    """The linear D = bf16(alpha * A . B^T + bias) with GELU and MXFP8 (E4M3)
    quantization of the result fused into the epilogue; D is never written.
    Returns (y_codes u8 [M, N], y_scales u8 (E8M0, tile order)): the next
    linear's MXFP8 activation operand."""
    f = _fmt(fmt)
    dev = a_codes.device
    y_codes = y_codes if y_codes is not None else torch.empty((M, N), dtype=torch.uint8, device=dev)
    y_scales = y_scales if y_scales is not None else torch.empty(scale_bytes(MXFP8, M, N), dtype=torch.uint8,
                                                                 device=dev)
    _gemm_args(f, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias, M, N, K)
    _buf(y_codes, torch.uint8, codes_bytes(MXFP8, M, N), "y_codes")
    _buf(y_scales, torch.uint8, scale_bytes(MXFP8, M, N), "y_scales")
    _gemm_cuda(a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias, y_codes=y_codes, y_scales=y_scales)
    _check(_lib.block_scaled_linear_gelu_mxfp8(f, _ptr(a_codes), _ptr(a_scales), _ptr(a_global), _ptr(b_codes),
                                               _ptr(b_scales), _ptr(b_global), _ptr(bias), _ptr(y_codes),
                                               _ptr(y_scales), M, N, K, _stream(stream, dev)),
           "block_scaled_linear_gelu_mxfp8")
    return y_codes, y_scales


NVQ_ERR_SHAPE = -2
SHORT_M_FUSED_ROWS = 8      # QuantizedLinear's one-launch path: batches up to this many rows


def nvfp4_linear_short_m(x, b_codes, b_scales, b_global, N, bias=None, out=None, a_codes=None, a_scales=None,
                         a_global=None, stream=None):
    """The NVFP4 linear of a short batch (M <= 16) in one launch: the dynamic
    activation quantization and the block-scaled GEMM fused, bit for bit as
    nvfp4_quantize + block_scaled_linear.  a_codes / a_scales / a_global, if
    given, receive the activation's quantization.  Raises NvqError with code
    NVQ_ERR_SHAPE where the fused launch does not apply (then take the two
    calls)."""
    M, K = x.shape
    dev = x.device
    out = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    _mat(x, torch.bfloat16, M, K, "x")
    _buf(b_codes, torch.uint8, codes_bytes(NVFP4, N, K), "b_codes")
    _buf(b_scales, torch.uint8, scale_bytes(NVFP4, N, K), "b_scales")
    _buf(b_global, torch.float32, 4, "b_global")
    if bias is not None:
        _buf(bias, torch.bfloat16, 2 * N, "bias")
    _mat(out, torch.bfloat16, M, N, "out")
    if a_codes is not None:
        _buf(a_codes, torch.uint8, codes_bytes(NVFP4, M, K), "a_codes")
    if a_scales is not None:
        _buf(a_scales, torch.uint8, scale_bytes(NVFP4, M, K), "a_scales")
    if a_global is not None:
        _buf(a_global, torch.float32, 4, "a_global")
    _cuda(x=x, b_codes=b_codes, b_scales=b_scales, b_global=b_global, bias=bias, out=out, a_codes=a_codes,
          a_scales=a_scales, a_global=a_global)
    _check(_lib.nvfp4_linear_short_m(_ptr(x), M, K, _pitch(x), _ptr(b_codes), _ptr(b_scales), _ptr(b_global),
                                     _ptr(bias), _ptr(out), _pitch(out), N, _ptr(a_codes), _ptr(a_scales),
                                     _ptr(a_global), _stream(stream, dev)), "nvfp4_linear_short_m")
    return out


class QuantizedLinear:
    """A linear layer whose weight is quantized once (offline) and whose
    activations are quantized on every call, then multiplied on the
    block-scaled tensor cores.  Holds device buffers only; each call is the
    ABI sequence quantize -> block_scaled_linear on one stream.  The
    activation buffers (one set per batch size) are reused by every call, so
    calls on different streams must be ordered with respect to each other.
    MXFP8 activations take the weight's element type (E4M3, or E5M2 for
    "mxfp8_e5m2") and the floor exponent rule, as quantize_weight does.
    NVFP4 batches of at most 8 rows take the one-launch nvfp4_linear_short_m
    where it applies (same result, bit for bit; measured faster than the two
    calls up to 8 rows, slower at 16)."""

    def __init__(self, weight, fmt="nvfp4", bias=None):
        self.fmt = _fmt(fmt)
        self.N, self.K = weight.shape
        self.device = weight.device
        self.w_codes, self.w_scales, self.w_global = quantize_weight(self.fmt, weight)
        self.bias = bias
        self._ws = new_workspace(self.device) if self.fmt == NVFP4 else None
        self._bufs = {}
        self._short = {}        # batch size -> whether the fused short-M launch applies

    def _act_bufs(self, M):
        b = self._bufs.get(M)
        if b is None:
            cols = self.K // 2 if self.fmt == NVFP4 else self.K
            b = (torch.empty((M, cols), dtype=torch.uint8, device=self.device),
                 torch.empty(scale_bytes(self.fmt, M, self.K), dtype=torch.uint8, device=self.device),
                 torch.empty(1, dtype=torch.float32, device=self.device))
            self._bufs[M] = b
        return b

    def __call__(self, x, out=None, stream=None):
        M = x.shape[0]
        if self.fmt == NVFP4 and 0 < M <= SHORT_M_FUSED_ROWS and self._short.get(M, True):
            # one launch for a short batch where the split GEMM allows it
            try:
                return nvfp4_linear_short_m(x, self.w_codes, self.w_scales, self.w_global, self.N, bias=self.bias,
                                            out=out, stream=stream)
            except NvqError as e:
                if e.code != NVQ_ERR_SHAPE:
                    raise
                self._short[M] = False
        codes, scales, g = self._act_bufs(M)
        if self.fmt == NVFP4:
            nvfp4_quantize(x, codes, scales, g, workspace=self._ws, stream=stream)
        else:
            mxfp8_quantize(x, codes, scales, stream=stream, elem="e5m2" if self.fmt == MXFP8_E5M2 else "e4m3")
            g = None
        return block_scaled_linear(self.fmt, codes, scales, g, self.w_codes, self.w_scales, self.w_global,
                                   M, self.N, self.K, bias=self.bias, out=out, stream=stream)


# --------------------------------------------------------------------------- diagnostics

def device_status(stream=None, device=None):
    """Synchronize the stream; return and clear the device status word."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    rc = _lib.nvq_device_status(_stream(stream, dev))
    if rc < 0:
        raise NvqError(rc, "nvq_device_status")
    return rc


def probe_gelu(bits, stream=None):
    """Device BF16 GELU (the fused epilogue's) of BF16 bit patterns (int16/uint16 tensor)."""
    n = bits.numel()
    out = torch.empty(n, dtype=torch.int16, device=bits.device)
    _check(_lib.nvq_probe_gelu(_ptr(bits), n, _ptr(out), _stream(stream, bits.device)), "nvq_probe_gelu")
    return out


def set_wait_limit(limit_ns):
    """Test hook: limit (ns) of the kernels' pipeline waits for later launches
    in this process; 0 restores the defaults (nvq_set_wait_limit)."""
    _check(_lib.nvq_set_wait_limit(int(limit_ns)), "nvq_set_wait_limit")


def wait_limit():
    """The current limit (ns) of the kernels' pipeline waits; 0 = the defaults.
    Starts from NVQ_WAIT_LIMIT_NS in the environment (nvq_wait_limit)."""
    return int(_lib.nvq_wait_limit())


def probe_wait(limit_ns, device=None, stream=None):
    """Run the bounded-wait self-test; returns the nanoseconds the device waited
    (the status word then holds NVQ_STATUS_TIMEOUT; read it with device_status)."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    waited = torch.zeros(1, dtype=torch.int64, device=dev)
    _check(_lib.nvq_probe_wait(int(limit_ns), _ptr(waited), _stream(stream, dev)), "nvq_probe_wait")
    return int(waited.item())


def probe_bounds(device=None, stream=None):
    """Run the bounds-check self-test (one failing check, no memory access):
    in the debug build the status word then holds NVQ_STATUS_BOUNDS."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    _check(_lib.nvq_probe_bounds(_stream(stream, dev)), "nvq_probe_bounds")


def probe_convert(values, stream=None):
    """Device FP32 -> (E2M1 codes, E4M3 codes) with the quantizers' conversions."""
    n = values.numel()
    e2 = torch.empty(n, dtype=torch.uint8, device=values.device)
    e4 = torch.empty(n, dtype=torch.uint8, device=values.device)
    _check(_lib.nvq_probe_convert(_ptr(values), n, _ptr(e2), _ptr(e4), _stream(stream, values.device)),
           "nvq_probe_convert")
    return e2, e4
