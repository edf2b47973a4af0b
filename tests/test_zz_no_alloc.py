"""The quantizer entry point that allocates nothing (nvfp4_quantize_noalloc).

Some callers cannot call cudaMalloc or hand the library a workspace: code
inside a host framework that owns all device memory and gives its plug-ins
no allocator or scratch buffer, or code on a latency-critical path that must
not allocate.  For them the library offers a variant of the dynamic NVFP4
quantizer whose scratch (the amax pass's partial maxima) is a static array
inside the library.  Its results must be those of nvfp4_quantize with a
workspace, bit for bit, call after call: the shared scratch keeps the last
call's contents, so two calls in a row on different tensors also check that
nothing stale leaks from one call into the next.

This file is named to be collected last, and it works both on its own in a
fresh process (its first call is the first on the device) and after the
rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import bits

pytestmark = pytest.mark.gpu

nvq = pytest.importorskip("microscaling_quantized_linear_b200")


def quantize_noalloc_cabi(x):
    """Calls the C entry point directly with caller-allocated outputs (x may
    be a row-pitched view)."""
    M, K = x.shape
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty(nvq.scale_bytes("nvfp4", M, K), dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = nvq._lib.nvfp4_quantize_noalloc(ctypes.c_void_p(x.data_ptr()), M, K, x.stride(0),
                                         ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
                                         ctypes.c_void_p(g.data_ptr()), stream)
    assert rc == 0, nvq.status_string(rc)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), g.cpu().numpy()


def quantize_with_workspace(x):
    codes, scales, g = nvq.nvfp4_quantize(x, workspace=nvq.new_workspace())
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), g.cpu().numpy()


def assert_same(a, b):
    # codes, scales and global scale are integers / exactly rounded: bit-exact
    for u, v, name in zip(a, b, ("codes", "scales", "global scale")):
        assert u.shape == v.shape and np.array_equal(u.view(np.uint8), v.view(np.uint8)), name


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    # A large-amax tensor, then a small-amax one, then the first again: each
    # call of the no-alloc entry point must reproduce the workspace entry point.
    tensors = [workloads.activation("ffup").cuda(),                 # outliers x50
               workloads.normal(4608, 3072, seed=5, std=1e-3).cuda(),
               workloads.activation("tiny").cuda()]
    tensors.append(tensors[0])
    for x in tensors:
        first = quantize_noalloc_cabi(x)
        second = quantize_noalloc_cabi(x)
        want = quantize_with_workspace(x)
        assert_same(first, want)
        assert_same(second, want)
        assert_same(first, oracle_quantize(x.cpu()))
    assert nvq.device_status() == 0


def oracle_quantize(x_cpu):
    codes, sf, g = oracle.nvfp4_quantize(bits(x_cpu))
    return codes, sf, np.array([g], dtype=np.float32)


SHAPES = [
    # ragged row counts (the scale rows up to the next multiple of 128 are
    # written as zero), several CTAs' partial maxima, and a pitched view
    (129, 512, None),
    (1000, 1536, None),
    (256, 448, 448 + 64),
]


@pytest.mark.parametrize("M,K,ldx", SHAPES)
def test_noalloc_matches_oracle_on_ragged_and_pitched_inputs(M, K, ldx):
    x = workloads.normal(M, K, seed=M + K, std=2.0)
    if ldx is None:
        xd = x.cuda()
    else:
        buf = torch.zeros((M, ldx), dtype=torch.bfloat16)
        buf[:, :K] = x
        xd = buf.cuda()[:, :K]
    want = oracle_quantize(x)
    assert_same(quantize_noalloc_cabi(xd), want)
    assert_same(quantize_noalloc_cabi(xd), want)           # second call on the same scratch
    assert_same(quantize_with_workspace(xd), want)
    assert nvq.device_status() == 0


def test_noalloc_python_wrapper_and_nonfinite_status():
    # The package's wrapper passes caller-allocated outputs to the same entry
    # point; an infinity in the input sets NVQ_STATUS_NONFINITE, and the next
    # finite call is clean and exact again.
    x = workloads.activation("ffup", seed=3)
    M, K = x.shape
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty(nvq.scale_bytes("nvfp4", M, K), dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    bad = x.clone()
    bad[17, 5] = float("inf")
    nvq.nvfp4_quantize_noalloc(bad.cuda(), codes, scales, g)
    assert nvq.device_status() == nvq.NVQ_STATUS_NONFINITE
    nvq.nvfp4_quantize_noalloc(x.cuda(), codes, scales, g)
    assert nvq.device_status() == 0
    assert_same((codes.cpu().numpy(), scales.cpu().numpy(), g.cpu().numpy()), oracle_quantize(x))


def test_noalloc_rejects_bad_arguments_without_launching():
    x = workloads.activation("tiny").cuda()
    M, K = x.shape
    null = ctypes.c_void_p(0)
    rc = nvq._lib.nvfp4_quantize_noalloc(ctypes.c_void_p(x.data_ptr()), M, K - 16, K, null, null, null, null)
    assert rc == -2                      # K not a multiple of 64
    rc = nvq._lib.nvfp4_quantize_noalloc(ctypes.c_void_p(x.data_ptr()), M, K, K, null, null, null, null)
    assert rc == -1                      # outputs must be given
