"""Quantize + GEMM replayed from CUDA graphs, with new activations every replay.

The batch-1 configuration on the pages runs the transformer under CUDA graphs
(page "Modelos de Difusão", FLUX.1-dev benchmark parameters: batch size 1
compiled with mode='reduce-overhead').  A captured launch keeps its
arguments, so any per-call state of the library has to live on the device:
the one-pass NVFP4 quantizer's grid barrier tags its slots from a generation
word in the workspace for exactly this reason.  The test captures the FF-up
step (dynamic NVFP4 quantization of [4608, 3072], the one-pass kernel, then
the block-scaled GEMM against the [12288, 3072] weight) in two graphs, and
mixes their replays with eager calls on the same workspace, copying a
different seeded activation into the captured input buffer before each one
(among them one whose amax is 2^-10 times smaller).  Codes, scales and the
global scale must equal the oracle's bit for bit after every replay, and the
GEMM output must meet the tolerance on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import bits, check_gemm, wgt

pytestmark = pytest.mark.gpu

nvq = pytest.importorskip("microscaling_quantized_linear_b200")


def replay_inputs(M, K):
    xs = []
    for i in range(12):
        x = workloads.activation("ffup", seed=300 + i)
        if i == 3:
            x = (x.float() * 2.0 ** -10).to(torch.bfloat16)      # a much smaller amax
        if i == 6:
            x = workloads.activation("actq", seed=301)            # per-channel scales
        if i == 9:
            x = x.clone()
            x[4321, 77] = 3000.0                                  # one large outlier
        xs.append(x)
    return xs


def test_graph_replays_match_oracle_every_time():
    w = wgt("ffup")
    N, K = w.shape
    M = 4608
    wc, wsf, wg = nvq.quantize_weight("nvfp4", w.cuda())
    B = oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(bits(w)), N, K)

    x_buf = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty(nvq.scale_bytes("nvfp4", M, K), dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = nvq.new_workspace()
    xs = replay_inputs(M, K)
    s = torch.cuda.Stream()

    def step():
        nvq.nvfp4_quantize(x_buf, codes, scales, g, workspace=ws, stream=s)
        nvq.block_scaled_linear("nvfp4", codes, scales, g, wc, wsf, wg, M, N, K, out=out, stream=s)

    with torch.cuda.stream(s):
        x_buf.copy_(xs[0].cuda())
        step()                                   # first call: per-device set-up before any capture
        s.synchronize()
        graphs = {}
        for name in ("A", "B"):
            graphs[name] = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graphs[name], stream=s):
                step()
            s.synchronize()

    # replays of both graphs and eager calls, interleaved on one workspace
    plan = ["A", "A", "eager", "A", "B", "B", "A", "eager", "B", "A", "A", "B"]
    rng = np.random.default_rng(12)
    for i, how in enumerate(plan):
        x = xs[i]
        with torch.cuda.stream(s):
            x_buf.copy_(x.cuda())
            if how == "eager":
                step()
            else:
                graphs[how].replay()
        s.synchronize()
        assert nvq.device_status() == 0, (i, how)
        oc, osf, og = oracle.nvfp4_quantize(bits(x))
        gc = codes.cpu().numpy()
        assert np.array_equal(gc, oc), "%s replay %d: %d code bytes differ" % (how, i, int((gc != oc).sum()))
        assert np.array_equal(scales.cpu().numpy(), osf), "%s replay %d: scales differ" % (how, i)
        assert np.float32(g.item()).tobytes() == np.float32(og).tobytes(), (how, i, g.item(), og)
        if i % 4 == 3:
            rows = np.sort(np.concatenate([[0, M - 1], rng.integers(0, M, 14)]))
            A = oracle.nvfp4_dequantize(oc, osf, og, M, K)
            Y = oracle.gemm_rows(A, B, rows=rows)
            check_gemm(out.float().cpu().numpy()[rows], Y)
    del graphs
