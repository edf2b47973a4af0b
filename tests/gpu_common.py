"""Shared helpers for the GPU parity tests (inputs from workloads, expected
values from the oracle only)."""
import functools

import numpy as np
import torch

import oracle
import workloads


def bits(x_bf16):
    return x_bf16.contiguous().view(torch.int16).numpy().view(np.uint16)


def sf_matrix(sf, rows, cols):
    """Logical [rows, cols] view of a tile-ordered scale buffer (numpy)."""
    r = np.arange(rows)[:, None]
    c = np.arange(cols)[None, :]
    off = ((r // 128) * ((cols + 3) // 4) + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (c % 4)
    return np.asarray(sf)[off]


@functools.lru_cache(maxsize=16)
def act(name, seed=0, M=None, K=None):
    return workloads.activation(name, seed=seed, M=M, K=K)


@functools.lru_cache(maxsize=16)
def wgt(name, seed=1):
    return workloads.weight(name, seed=seed)


@functools.lru_cache(maxsize=32)
def oracle_nvfp4(key, x_fn):
    return oracle.nvfp4_quantize(bits(x_fn()))


def sample_rows(M, seed=2, per_tile_every=1, extra=32):
    """First and last row of every `per_tile_every`-th 128-row tile, plus random rows."""
    rows = set()
    for t in range(0, M // 128, per_tile_every):
        rows.add(128 * t)
        rows.add(128 * t + 127)
    rng = np.random.default_rng(seed)
    rows.update(rng.integers(0, M, extra).tolist())
    return np.array(sorted(rows), dtype=np.int64)


def check_gemm(D, Y, tol=oracle.GEMM_TOL):
    err = oracle.gemm_row_errors(D, Y)
    worst = int(np.argmax(err))
    assert err.max() <= tol, "row %d: rel err %.3e > %.1e" % (worst, err.max(), tol)
    return float(err.max())
