"""Failure detection on the GPU without a fault: bounded waits that run out.

Every wait between the roles of a kernel is bounded in wall time; when one
gives up, the kernel sets NVQ_STATUS_TIMEOUT in the device status word and
returns, so the context stays usable.  nvq_probe_wait runs that bounded wait
on an mbarrier nothing arrives on (a flag that nothing sets).  The test hook
nvq_set_wait_limit shortens the real kernels' waits so that they run out: the
one-CTA GEMM's pipeline waits and the one-pass quantizer's grid barrier and the split-K
cluster's exchange.  The tests read the status on the host and then check
that the context still computes correct results.  Nothing faults, traps or
hangs: every kernel still waits, with its usual 4 s limit, for its own
copies and tensor-core work before it exits, and a split-K CTA for every
push into its shared memory.  (The CTA-pair GEMM's abort path is not driven
here: its peer CTA's loads complete on the leader's barriers.)
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


def test_one_pass_quantizer_barrier_wait_runs_out_results_stay_exact():
    # [4608, 3072] takes the one-pass kernel, whose CTAs wait for each
    # other's partial maxima.  With a 1 ns limit the first CTAs to publish
    # give up at once: they report NVQ_STATUS_TIMEOUT and read the amax from
    # the whole tensor themselves, so every output stays exact.
    x = workloads.activation("actq")
    y = workloads.activation("actq", seed=7)
    xd, yd = x.cuda(), y.cuda()
    ws = nvq.new_workspace()
    assert nvq.device_status() == 0
    nvq.set_wait_limit(1)
    try:
        got = nvq.nvfp4_quantize(xd, workspace=ws)
        status = nvq.device_status()
    finally:
        nvq.set_wait_limit(0)
    assert status == nvq.NVQ_STATUS_TIMEOUT
    for gpu, want in zip(got, oracle.nvfp4_quantize(bits(x))):
        assert np.array_equal(gpu.cpu().numpy().reshape(-1).view(np.uint8), np.asarray(want).reshape(-1).view(np.uint8))
    # the same workspace, default limit: a clean, exact call on another tensor
    got = nvq.nvfp4_quantize(yd, workspace=ws)
    assert nvq.device_status() == 0
    for gpu, want in zip(got, oracle.nvfp4_quantize(bits(y))):
        assert np.array_equal(gpu.cpu().numpy().reshape(-1).view(np.uint8), np.asarray(want).reshape(-1).view(np.uint8))


def test_gemm_pipeline_wait_runs_out_and_the_context_survives():
    # The tiny linear runs on the one-CTA kernel (one 128 x 128 tile).  With a
    # 1 ns limit the MMA lane's first wait for its operands gives up: the
    # kernel raises NVQ_STATUS_TIMEOUT, every role leaves its loop, the CTA
    # waits (bounded) for its own loads and tensor-core work, frees tensor
    # memory and returns.  The output is then unspecified; the next call, at
    # the default limit, must be clean and match the oracle.
    x, w = workloads.activation("tiny"), workloads.weight("tiny")
    M, K = x.shape
    N = w.shape[0]
    assert nvq.gemm_plan("nvfp4", M, N, K) == (128, 128, 1)
    ac, as_, ag = nvq.nvfp4_quantize(x.cuda())
    wc, ws, wg = nvq.quantize_weight("nvfp4", w.cuda())
    assert nvq.device_status() == 0
    nvq.set_wait_limit(1)
    try:
        nvq.block_scaled_linear("nvfp4", ac, as_, ag, wc, ws, wg, M, N, K)
        status = nvq.device_status()
    finally:
        nvq.set_wait_limit(0)
    assert status == nvq.NVQ_STATUS_TIMEOUT
    D = nvq.block_scaled_linear("nvfp4", ac, as_, ag, wc, ws, wg, M, N, K)
    assert nvq.device_status() == 0
    oc, os_, og = oracle.nvfp4_quantize(bits(x))
    Y = oracle.gemm_rows(oracle.nvfp4_dequantize(oc, os_, og, M, K),
                         oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(bits(w)), N, K))
    check_gemm(D.float().cpu().numpy(), Y)


def test_split_k_waits_run_out_and_the_context_survives():
    # The FF-up weight at M = 1 runs as clusters of two CTAs, each over half
    # of K.  With a 1 ns limit the pipeline waits give up; the epilogue warps
    # still send their (unspecified) slots, so every CTA's wait for the
    # cluster's copies ends, and no CTA exits while a copy into or out of its
    # shared memory is in flight.  The next call, at the default limit, must
    # be clean and match the oracle.
    w = workloads.weight("ffup")
    N, K = w.shape
    x = workloads.activation("ffup", seed=5, M=1)
    M = 1
    tm, tn, ks = nvq.gemm_plan("nvfp4", M, N, K)
    assert ks > 1
    ac, as_, ag = nvq.nvfp4_quantize(x.cuda())
    wc, ws, wg = nvq.quantize_weight("nvfp4", w.cuda())
    assert nvq.device_status() == 0
    nvq.set_wait_limit(1)
    try:
        for _ in range(3):
            nvq.block_scaled_linear("nvfp4", ac, as_, ag, wc, ws, wg, M, N, K)
        status = nvq.device_status()
    finally:
        nvq.set_wait_limit(0)
    assert status == nvq.NVQ_STATUS_TIMEOUT
    D = nvq.block_scaled_linear("nvfp4", ac, as_, ag, wc, ws, wg, M, N, K)
    assert nvq.device_status() == 0
    oc, os_, og = oracle.nvfp4_quantize(bits(x))
    Y = oracle.gemm_rows(oracle.nvfp4_dequantize(oc, os_, og, M, K),
                         oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(bits(w)), N, K))
    check_gemm(D.float().cpu().numpy(), Y)
