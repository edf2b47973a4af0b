"""Host-side checks of the C-ABI library that need no GPU.

The library loads without a GPU driver, exports every entry point that
include/nvq.h declares, and rejects bad arguments before touching the device
(no kernel is launched and no pointer is dereferenced on these paths).
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import microscaling_quantized_linear_b200 as nvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvq.h")

NULL = None
P16 = ctypes.c_void_p(0x10000)         # aligned, never dereferenced
P_ODD = ctypes.c_void_p(0x10008)       # 8-byte aligned only
L = nvq._lib


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^NVQ_API\s+[\w\s\*]*?\b(\w+)\s*\(", src, re.M)))


def test_header_declarations_are_all_exported():
    declared = declared_functions()
    assert len(declared) >= 10
    out = subprocess.run(["nm", "-D", "--defined-only", nvq.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [f for f in declared if f not in exported]
    assert not missing, missing
    assert set(declared) == set(nvq.EXPORTED)


def test_library_links_no_cuda_shared_objects():
    out = subprocess.run(["ldd", nvq.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda" not in out and "libcudart" not in out


def test_size_helpers():
    assert nvq.codes_bytes("nvfp4", 4608, 3072) == 4608 * 1536
    assert nvq.codes_bytes("mxfp8", 4608, 12288) == 4608 * 12288
    assert nvq.scale_bytes("nvfp4", 4608, 3072) == 4608 * 192
    assert nvq.scale_bytes("mxfp8", 4608, 12288) == 4608 * 384
    assert nvq.scale_bytes("nvfp4", 130, 80) == 256 * 8          # padded to 128 rows x 4 columns
    assert nvq.scale_bytes("mxfp8_e5m2", 100, 256) == nvq.scale_bytes("mxfp8", 100, 256) == 128 * 8
    assert nvq.codes_bytes("mxfp8_e5m2", 100, 256) == 100 * 256
    assert nvq.workspace_bytes() >= 4 * 148
    assert L.nvq_codes_bytes(7, 128, 64) == 0


def test_status_strings():
    for code in (0, -1, -2, -3, -4, -5, -7):
        assert nvq.status_string(code) and nvq.status_string(code) != "unknown status"


def q4(x=P16, M=128, K=64, ld=64, codes=P16, scales=P16, g=P16, calib=NULL, ws=P16):
    return L.nvfp4_quantize(x, M, K, ld, codes, scales, g, calib, ws, NULL)


def test_nvfp4_quantize_rejects_bad_arguments():
    assert q4(x=NULL) == -1
    assert q4(codes=NULL) == -1
    assert q4(g=NULL) == -1
    assert q4(ws=NULL) == -1                 # dynamic path needs the workspace
    assert q4(K=48, ld=48) == -2             # K not a multiple of 64
    assert q4(ld=60) == -2                   # pitch < K
    assert q4(ld=68) == -2                   # pitch not a multiple of 8
    assert q4(M=-128) == -2
    assert q4(M=1 << 20, K=1 << 12, ld=1 << 12) == -2   # rows * K >= 2^31
    assert q4(x=P_ODD) == -3
    assert q4(codes=P_ODD) == -3


def test_mxfp8_quantize_rejects_bad_arguments():
    assert L.mxfp8_quantize(NULL, 128, 128, 128, P16, P16, NULL) == -1
    assert L.mxfp8_quantize(P16, 128, 64, 64, P16, P16, NULL) == -2      # K not a multiple of 128
    assert L.mxfp8_quantize(P16, 128, 128, 128, P_ODD, P16, NULL) == -3


def test_mxfp8_quantize_ex_rejects_bad_arguments():
    def qx(elem=1, rule=0, x=P16, M=128, K=128, codes=P16):
        return L.mxfp8_quantize_ex(x, M, K, K, codes, P16, elem, rule, NULL)
    assert qx(elem=0) == -7                   # NVFP4 is not an MXFP8 element type
    assert qx(elem=3) == -7
    assert qx(rule=2) == -7
    assert qx(x=NULL) == -1
    assert qx(K=64) == -2
    assert qx(codes=P_ODD) == -3


def test_quantize_weight_rejects_bad_format():
    assert L.quantize_weight(5, P16, 128, 64, 64, P16, P16, P16, P16, NULL) == -7


def gemm(fmt=0, a=P16, sa=P16, ga=P16, b=P16, sb=P16, gb=P16, bias=NULL, out=P16, ldo=128, M=128, N=128, K=256):
    return L.block_scaled_linear(fmt, a, sa, ga, b, sb, gb, bias, out, ldo, M, N, K, NULL)


def test_block_scaled_linear_rejects_bad_arguments():
    assert gemm(fmt=3) == -7
    assert gemm(M=-1) == -2
    assert gemm(a=NULL) == -1
    assert gemm(ga=NULL) == -1                # NVFP4 needs both global scales
    assert gemm(out=NULL) == -1
    assert gemm(N=0, ldo=8) == -2
    assert gemm(N=130, ldo=136) == -2          # N must be a multiple of 8
    assert gemm(K=96) == -2
    assert gemm(K=192) == -2                  # NVFP4 GEMM K must be a multiple of 256
    assert gemm(fmt=1, ga=NULL, gb=NULL, K=64) == -2     # MXFP8 K must be a multiple of 128
    assert gemm(ldo=120) == -2
    assert gemm(ldo=132) == -2
    assert gemm(a=P_ODD) == -3
    assert gemm(out=P_ODD) == -3


def gemm_gelu(fmt=0, a=P16, sa=P16, ga=P16, b=P16, sb=P16, gb=P16, bias=NULL, yc=P16, ys=P16, M=128, N=128,
              K=256):
    return L.block_scaled_linear_gelu_mxfp8(fmt, a, sa, ga, b, sb, gb, bias, yc, ys, M, N, K, NULL)


def test_block_scaled_linear_gelu_mxfp8_rejects_bad_arguments():
    assert gemm_gelu(fmt=2) == -7             # E5M2 operands are not offered here
    assert gemm_gelu(fmt=5) == -7
    assert gemm_gelu(M=-1) == -2
    assert gemm_gelu(N=64) == -2               # N (the next layer's K) must be a multiple of 128
    assert gemm_gelu(N=136) == -2
    assert gemm_gelu(K=128) == -2              # NVFP4 K must be a multiple of 256
    assert gemm_gelu(fmt=1, ga=NULL, gb=NULL, K=64) == -2
    assert gemm_gelu(yc=NULL) == -1
    assert gemm_gelu(ys=NULL) == -1
    assert gemm_gelu(gb=NULL) == -1
    assert gemm_gelu(yc=P_ODD) == -3
    assert gemm_gelu(ys=P_ODD) == -3
    assert gemm_gelu(M=0) == 0                 # empty batch: nothing to do
    assert L.nvq_probe_gelu(NULL, 4, P16, NULL) == -1
    assert L.nvq_probe_wait(1000, NULL, NULL) == -1
    assert L.nvq_probe_wait(2 * 10**9, P16, NULL) == -2
    assert L.nvq_probe_gelu(P16, -1, P16, NULL) == -2


def test_gemm_plan_rejects_bad_arguments():
    def plan(fmt=0, M=1, N=12288, K=3072, tm=P16, tn=P16, ks=P16):
        return L.nvq_gemm_plan(fmt, M, N, K, tm, tn, ks)
    assert plan(fmt=3) == -7
    assert plan(tm=NULL) == -1
    assert plan(ks=NULL) == -1
    assert plan(M=0) == -2                     # a plan needs at least one row
    assert plan(N=12) == -2
    assert plan(K=128) == -2                   # NVFP4 K must be a multiple of 256
    assert plan(fmt=1, K=64) == -2


def test_valid_arguments_without_gpu_report_cuda_error():
    # Arguments pass the host checks; with no device the library reports a
    # CUDA error instead of launching.
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert q4() == -5
    assert gemm() == -5
    # ragged row counts pass the host checks (the scale tiles are padded)
    assert q4(M=100) == -5
    assert gemm(M=96, N=64, ldo=64) == -5
    assert gemm(fmt=2, ga=NULL, gb=NULL, K=128) == -5
    assert L.mxfp8_quantize_ex(P16, 100, 128, 128, P16, P16, 2, 1, NULL) == -5
    assert gemm_gelu() == -5
    assert gemm_gelu(fmt=1, ga=NULL, gb=NULL, M=100, N=384, K=128) == -5
    assert L.nvq_probe_gelu(P16, 16, P16, NULL) == -5
    assert L.nvq_probe_wait(1000, P16, NULL) == -5
    out = (ctypes.c_int * 3)()
    assert L.nvq_gemm_plan(0, 1, 12288, 3072, ctypes.byref(out, 0), ctypes.byref(out, 4),
                           ctypes.byref(out, 8)) == -5


def test_wait_limit_hook_and_workspace_init_check_arguments():
    # the test hook only stores a process-wide limit: no device needed
    assert L.nvq_set_wait_limit(4_000_000_001) == -2        # above the 4 s default
    assert L.nvq_set_wait_limit(1000) == 0
    assert L.nvq_set_wait_limit(0) == 0                     # back to the defaults
    assert L.nvq_workspace_init(NULL, NULL) == -1
    assert L.nvq_workspace_init(P_ODD, NULL) == -3
    # the workspace holds the one-pass slots (one 128-byte line per CTA, up to
    # 256), the two-pass partials and the generation word's line
    assert nvq.workspace_bytes() == 256 * 128 + 1024 * 4 + 128


def test_binding_checks_buffers_before_the_library_sees_them():
    # The C ABI takes raw pointers and cannot check what they point to; the
    # binding checks dtype, contiguity and size (then the device) first.
    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    u8 = lambda n: torch.zeros(n, dtype=torch.uint8)
    f32 = lambda n: torch.zeros(n, dtype=torch.float32)
    M, K = 128, 256
    with pytest.raises(ValueError, match="x: expected torch.bfloat16"):
        nvq.nvfp4_quantize(torch.zeros(M, K), u8(M * K // 2), u8(nvq.scale_bytes("nvfp4", M, K)), f32(1))
    with pytest.raises(ValueError, match="codes: .* the call needs 16384"):
        nvq.nvfp4_quantize(bf(M, K), u8(100), u8(nvq.scale_bytes("nvfp4", M, K)), f32(1))
    with pytest.raises(ValueError, match="scales: .* the call needs"):
        nvq.nvfp4_quantize_noalloc(bf(M, K), u8(M * K // 2), u8(8), f32(1))
    with pytest.raises(ValueError, match="global_scale: expected torch.float32"):
        nvq.nvfp4_quantize(bf(M, K), u8(M * K // 2), u8(nvq.scale_bytes("nvfp4", M, K)), u8(4))
    with pytest.raises(ValueError, match="workspace: .* the call needs"):
        nvq.nvfp4_quantize(bf(M, K), u8(M * K // 2), u8(nvq.scale_bytes("nvfp4", M, K)), f32(1), workspace=u8(16))
    with pytest.raises(ValueError, match="codes: expected a contiguous tensor"):
        nvq.mxfp8_quantize(bf(M, K), torch.zeros(M, 2 * K, dtype=torch.uint8)[:, ::2], u8(4096))
    with pytest.raises(ValueError, match="w: expected a \\[256, 128\\] matrix with unit column stride"):
        nvq.quantize_weight("mxfp8", bf(M, K).t(), u8(M * K), u8(nvq.scale_bytes("mxfp8", M, K)))
    ops = dict(a_codes=u8(M * K // 2), a_scales=u8(nvq.scale_bytes("nvfp4", M, K)), a_global=f32(1),
               b_codes=u8(M * K // 2), b_scales=u8(nvq.scale_bytes("nvfp4", M, K)), b_global=f32(1))
    with pytest.raises(ValueError, match="out: expected a \\[128, 128\\] matrix"):
        nvq.block_scaled_linear("nvfp4", M=M, N=M, K=K, out=bf(M, 64), **ops)
    with pytest.raises(ValueError, match="bias: .* the call needs 256"):
        nvq.block_scaled_linear("nvfp4", M=M, N=M, K=K, bias=bf(64), out=bf(M, M), **ops)
    with pytest.raises(ValueError, match="NVFP4 operands need their global scales"):
        nvq.block_scaled_linear("nvfp4", M=M, N=M, K=K, out=bf(M, M), **dict(ops, a_global=None))
    with pytest.raises(ValueError, match="y_codes: .* the call needs"):
        nvq.block_scaled_linear_gelu_mxfp8("nvfp4", M=M, N=M, K=K, y_codes=u8(10), y_scales=u8(1 << 14), **ops)
    # right dtypes and sizes on the host: only the device is wrong
    with pytest.raises(ValueError, match="expected a CUDA tensor"):
        nvq.block_scaled_linear("nvfp4", M=M, N=M, K=K, out=bf(M, M), **ops)


def test_linear_short_m_rejects_bad_arguments():
    def ls(x=P16, M=1, K=256, ldx=256, b=P16, sb=P16, gb=P16, bias=NULL, out=P16, ldo=128, N=128):
        return L.nvfp4_linear_short_m(x, M, K, ldx, b, sb, gb, bias, out, ldo, N, NULL, NULL, NULL, NULL)
    assert ls(M=17) == -2                     # short batches only
    assert ls(K=192, ldx=192) == -2           # K a multiple of 256
    assert ls(N=100, ldo=104) == -2           # N a multiple of 8
    assert ls(ldo=120) == -2
    assert ls(x=NULL) == -1
    assert ls(gb=NULL) == -1
    assert ls(out=P_ODD) == -3
    assert ls(M=0) == 0                       # empty batch: nothing to do


def test_wait_limit_starts_from_the_environment():
    # NVQ_WAIT_LIMIT_NS sets the initial limit when the library loads; a
    # malformed or too large value leaves the defaults (0).  Host only.
    import subprocess
    import sys
    code = ("import sys; sys.path.insert(0, %r); import microscaling_quantized_linear_b200 as n; "
            "print(n.wait_limit())" % os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    got = {}
    for val in ("12345", "4000000000", "4000000001", "12x", ""):
        env = dict(os.environ, NVQ_WAIT_LIMIT_NS=val)
        out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
        assert out.returncode == 0, out.stderr[-2000:]
        got[val] = int(out.stdout.strip().splitlines()[-1])
    assert got == {"12345": 12345, "4000000000": 4000000000, "4000000001": 0, "12x": 0, "": 0}
    assert L.nvq_set_wait_limit(777) == 0
    assert nvq.wait_limit() == 777
    assert L.nvq_set_wait_limit(0) == 0
    assert nvq.wait_limit() == 0
