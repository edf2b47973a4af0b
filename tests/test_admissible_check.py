"""CPU checks of the fused epilogue's admissibility test (tests/admissible.py):
it accepts the oracle's own outputs and rejects planted mistakes."""
import numpy as np
import pytest

import oracle
import workloads
from admissible import check_admissible
from gpu_common import bits, sf_matrix


def test_admissible_check_rejects_wrong_bytes():
    # The check itself, on the oracle's own outputs (accepted) and on planted
    # mistakes (rejected): a scale byte two exponents off, a code four steps
    # off, a sign flipped.
    x = workloads.activation("ffup", seed=4, M=128, K=512)
    w = workloads.weight("ffup", seed=5, N=1024, K=512)
    xq, wq = oracle.nvfp4_quantize(bits(x)), oracle.nvfp4_quantize(bits(w))
    A = oracle.nvfp4_dequantize(*xq, 128, 512)
    B = oracle.nvfp4_dequantize(*wq, 1024, 512)
    oc, osf, _, _, Y = oracle.linear_gelu_mxfp8(A, B)
    ys = sf_matrix(osf, 128, 32)
    check_admissible(oc, ys, Y)
    bad_s = ys.copy()
    bad_s[5, 7] += 2
    with pytest.raises(AssertionError, match="scale"):
        check_admissible(oc, bad_s, Y)
    big = np.argwhere((oc & 0x7F) > 0x30)[0]
    for planted in ((oc[tuple(big)] & 0x80) | ((oc[tuple(big)] & 0x7F) - 4), oc[tuple(big)] ^ 0x80):
        bad_c = oc.copy()
        bad_c[tuple(big)] = planted
        with pytest.raises(AssertionError, match="codes"):
            check_admissible(bad_c, ys, Y)
