"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every pipeline wait in the GEMM kernels is bounded in wall time; when one
gives up, the kernel sets NVQ_STATUS_TIMEOUT in the device status word and
returns, so the context stays usable.  nvq_probe_wait runs that same bounded
wait on an mbarrier nothing arrives on (a flag that nothing sets); the test
reads the status on the host and then checks that the context still computes
correct results.  Nothing faults, traps or hangs.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import bits, check_gemm

pytestmark = pytest.mark.gpu

nvq = pytest.importorskip("microscaling_quantized_linear_b200")


def test_bounded_wait_gives_up_and_reports_timeout():
    assert nvq.device_status() == 0
    limit = 2_000_000                                      # 2 ms
    waited = nvq.probe_wait(limit)
    assert limit <= waited < 1_000_000_000
    assert nvq.device_status() == nvq.NVQ_STATUS_TIMEOUT
    assert nvq.device_status() == 0                        # read clears it
    # the context is intact: the tiny linear still matches the oracle
    x, w = workloads.activation("tiny"), workloads.weight("tiny")
    M, K = x.shape
    N = w.shape[0]
    ac, as_, ag = nvq.nvfp4_quantize(x.cuda())
    wc, ws, wg = nvq.quantize_weight("nvfp4", w.cuda())
    D = nvq.block_scaled_linear("nvfp4", ac, as_, ag, wc, ws, wg, M, N, K)
    assert nvq.device_status() == 0
    oc, os_, og = oracle.nvfp4_quantize(bits(x))
    assert np.array_equal(ac.cpu().numpy(), oc) and np.array_equal(as_.cpu().numpy(), os_)
    Y = oracle.gemm_rows(oracle.nvfp4_dequantize(oc, os_, og, M, K),
                         oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(bits(w)), N, K))
    check_gemm(D.float().cpu().numpy(), Y)


def test_zero_limit_gives_up_at_once():
    waited = nvq.probe_wait(0)
    assert waited < 100_000_000
    assert nvq.device_status() == nvq.NVQ_STATUS_TIMEOUT
