"""Seeded synthetic inputs for the microscaling-quantized linear layer.

This module only draws random numbers; it holds none of the quantization or
GEMM arithmetic.  Both the CUDA path's tests/benchmark and the CPU oracle's
tests take their inputs from here.

The shapes are those of FLUX.1-dev's transformer linears at 1024x1024: 64x64
image tokens (1024 / VAE factor 8 / patch 2) plus 512 text tokens give
M = 4608 rows per image (page "NVIDIA量化推理：5步极速优化显存+成功率翻倍",
step 3 call parameters: height/width 1024, max_sequence_length 512).  The
hidden sizes 3072 / 9216 / 12288 are FLUX's model width, fused QKV width and
MLP width.  The value distributions stand in for the diffusion model's real
activations and weights, which are not available here:

  tiny   A [128, 256]   N(0,1), 1% of entries (Bernoulli mask) x20
         W [128, 256]   N(0, 0.02)
  actq   A [4608, 3072] N(0,1) * c_k per column, c_k ~ LogNormal(0, 1)
  ffup   A [4608, 3072] N(0,1), 0.5% of entries x50;  W [12288, 3072] N(0, 0.02)
  ffdown A [4608, 12288] GELU(N(0,1)) (exact erf form); W [3072, 12288] N(0, 0.01)
  qkv4   A [18432, 3072] 0.5 * StudentT(df=3);        W [9216, 3072] N(0, 0.02)

Each tensor is drawn in FP32 on the host with torch.Generator(seed) and
rounded to BF16 (round-to-nearest-even).  Activations use seed 0 (1 for the
weights, 2 for an optional bias ~ N(0, 0.1)); a different seed can be passed
to draw fresh tensors of the same recipe.
"""
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    fmt: str            # "nvfp4" or "mxfp8"
    M: int
    N: int
    K: int
    desc: str


WORKLOADS = {
    "tiny": Workload("tiny", "nvfp4", 128, 128, 256,
                     "NVFP4 W4A4 linear 128x128x256, A N(0,1) with 1% x20 outliers, W N(0,0.02)"),
    "actq": Workload("actq", "nvfp4", 4608, 0, 3072,
                     "NVFP4 activation quantization [4608,3072], N(0,1) x LogNormal(0,1) per channel"),
    "ffup": Workload("ffup", "nvfp4", 4608, 12288, 3072,
                     "NVFP4 W4A4 FF-up linear 4608x12288x3072 (FLUX-like), A N(0,1) 0.5% x50, W N(0,0.02)"),
    "ffdown": Workload("ffdown", "mxfp8", 4608, 3072, 12288,
                       "MXFP8 E4M3 FF-down linear 4608x3072x12288, A GELU(N(0,1)), W N(0,0.01)"),
    "qkv4": Workload("qkv4", "nvfp4", 18432, 9216, 3072,
                     "NVFP4 QKV projection at batch 4, 18432x9216x3072, A 0.5*StudentT(3), W N(0,0.02)"),
}


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _outliers(x, g, p, factor):
    mask = torch.rand(x.shape, generator=g) < p
    return torch.where(mask, x * factor, x)


def activation(name, seed=0, M=None, K=None):
    """BF16 activation tensor [M, K] of the named recipe (CPU)."""
    w = WORKLOADS[name]
    M = M or w.M
    K = K or w.K
    g = _gen(seed)
    if name == "tiny":
        x = _outliers(torch.randn(M, K, generator=g), g, 0.01, 20.0)
    elif name == "actq":
        c = torch.exp(torch.randn(1, K, generator=g))
        x = torch.randn(M, K, generator=g) * c
    elif name == "ffup":
        x = _outliers(torch.randn(M, K, generator=g), g, 0.005, 50.0)
    elif name == "ffdown":
        x = torch.nn.functional.gelu(torch.randn(M, K, generator=g), approximate="none")
    elif name == "qkv4":
        # Student-t with 3 degrees of freedom: Z / sqrt(V / 3), V ~ chi^2(3).
        z = torch.randn(M, K, generator=g)
        v = (torch.randn(3, M, K, generator=g) ** 2).sum(0)
        x = 0.5 * z / torch.sqrt(v / 3.0)
    else:
        raise KeyError(name)
    return x.to(torch.bfloat16)


def weight(name, seed=1, N=None, K=None):
    """BF16 weight tensor [N, K] of the named recipe (CPU)."""
    w = WORKLOADS[name]
    N = N or w.N
    K = K or w.K
    std = {"tiny": 0.02, "ffup": 0.02, "ffdown": 0.01, "qkv4": 0.02}[name]
    return (torch.randn(N, K, generator=_gen(seed)) * std).to(torch.bfloat16)


def bias(N, seed=2):
    """BF16 bias vector [N] ~ N(0, 0.1) (CPU)."""
    return (torch.randn(N, generator=_gen(seed)) * 0.1).to(torch.bfloat16)


def exact_operand(rows, K, seed, significands=(1.0, 1.5, 1.75), top_row=None, min_exp=-3, block=16):
    """BF16 [rows, K] whose values are c_r * e with e drawn from {0, +-0.5,
    +-1, +-1.5, +-2, +-3, +-4, +-6} and every `block` consecutive values of a
    row holding one +-6 * c_r; the row constants c_r = s * 2^i take s from
    `significands` and i from [min_exp, 0].  If top_row is given, that row's
    constant is 1.75 (the tensor's largest).  Returns (x, c) with c the
    binary64 row constants.  Products and sums of such values stay on a
    coarse binary grid, which makes a GEMM over them exact in binary32 for
    moderate K (CPU)."""
    g = _gen(seed)
    mags = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    e = mags[torch.randint(0, 8, (rows, K), generator=g)]
    e = torch.where(torch.rand(rows, K, generator=g) < 0.5, -e, e)
    pos = torch.randint(0, block, (rows, K // block), generator=g) + torch.arange(0, K, block)
    sign6 = torch.where(torch.rand(rows, K // block, generator=g) < 0.5, -6.0, 6.0)
    e.scatter_(1, pos, sign6)
    sig = torch.tensor(significands, dtype=torch.float64)
    c = sig[torch.randint(0, len(significands), (rows,), generator=g)] * \
        torch.pow(2.0, torch.randint(min_exp, 1, (rows,), generator=g).double())
    if top_row is not None:
        c[top_row] = 1.75
    x = (e.double() * c[:, None]).to(torch.bfloat16)
    return x, c.numpy()


def grid_bias(N, seed=3):
    """BF16 bias [N] of k / 16 with k uniform in [-16, 16] (on the same coarse
    grid as exact_operand's products for its exponents >= -3) (CPU)."""
    k = torch.randint(-16, 17, (N,), generator=_gen(seed))
    return (k.double() / 16.0).to(torch.bfloat16)


def normal(M, K, seed, std=1.0):
    """Plain BF16 N(0, std^2) tensor, for shape-sweep tests."""
    return (torch.randn(M, K, generator=_gen(seed)) * std).to(torch.bfloat16)
