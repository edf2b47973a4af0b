"""The GEMM planner on the host, with stated device facts (no GPU):
nvq_gemm_plan_host is the function nvq_gemm_plan evaluates with the current
device's SM count and resident-cluster limits.

The B200 facts are the ones cudaOccupancyMaxActiveClusters reported on a
B200 at one 416-thread CTA per SM: 74 clusters of 2, 45 of 3, 33 of 4, 26 of
5, 22 of 6 and 15 of 7 or 8 CTAs (148 SMs).
"""
import ctypes

import pytest

import microscaling_quantized_linear_b200 as nvq

SMS = 148
B200 = {(w, s): n for w in (128, 192, 256) for s, n in zip(range(2, 9), (74, 45, 33, 26, 22, 15, 15))}


def plan(fmt, M, N, K, facts=B200, sms=SMS, **kw):
    return nvq.gemm_plan_host(fmt, M, N, K, sms, facts, **kw)


@pytest.mark.parametrize("M", [1, 2, 16, 31, 32])
def test_ffup_weight_at_short_m_splits_on_192_wide_pairs_of_ctas(M):
    # 12288 / 128 = 96 CTAs unsplit; 48 clusters of three 256-wide CTAs would
    # need 48 > 45 resident clusters, so 64 clusters of two 192-wide CTAs
    # (128 SMs) win.
    assert plan("nvfp4", M, 12288, 3072) == (128, 192, 2)


def test_no_split_past_32_rows():
    assert plan("nvfp4", 33, 12288, 3072) == (128, 128, 1)
    assert plan("nvfp4", 128, 12288, 3072) == (128, 128, 1)


def test_pairs_above_one_row_block():
    assert plan("nvfp4", 129, 12288, 3072) == (256, 256, 1)
    assert plan("nvfp4", 4608, 12288, 3072) == (256, 256, 1)
    assert plan("mxfp8", 4608, 3072, 12288) == (256, 256, 1)
    assert plan("mxfp8_e5m2", 512, 1152, 384) == (256, 192, 1)   # N % 384 == 0, N % 256 != 0
    assert plan("nvfp4", 300, 520, 512) == (256, 256, 1)         # ragged N takes 256


def test_qkv_and_ffdown_widths():
    # QKV: 72 clusters of two 128-wide CTAs (144 SMs) beat 36 x 3 at 256
    assert plan("nvfp4", 32, 9216, 3072) == (128, 128, 2)
    # FF-down (K = 12288, 96 K stages): 24 clusters of five (120 SMs); six
    # would need 24 > 22 resident clusters
    assert plan("mxfp8", 24, 3072, 12288) == (128, 128, 5)


def test_switches():
    # without pairs the one-CTA kernel takes 256-wide tiles once they fill the SMs
    assert plan("nvfp4", 4608, 12288, 3072, use_pairs=False) == (128, 256, 1)
    assert plan("nvfp4", 64, 12288, 3072, use_pairs=False) == (128, 128, 1)
    assert plan("nvfp4", 1, 12288, 3072, use_splitk=False) == (128, 128, 1)


def test_split_needs_two_k_tiles_per_cta_and_resident_clusters():
    assert plan("nvfp4", 1, 12288, 256) == (128, 128, 1)       # one K stage
    assert plan("nvfp4", 1, 12288, 512) == (128, 128, 1)       # two: a split would leave one per CTA
    assert plan("nvfp4", 1, 12288, 1024) == (128, 192, 2)
    assert plan("nvfp4", 1, 12288, 3072, facts={}) == (128, 128, 1)   # no cluster fits
    # a device that holds 48 clusters of three: 144 SMs on 256-wide tiles
    more = dict(B200)
    more.update({(256, 3): 48})
    assert plan("nvfp4", 1, 12288, 3072, facts=more) == (128, 256, 3)


def test_split_must_add_a_quarter_more_sms():
    # only 2-clusters of 256-wide tiles fit: 96 CTAs, no more than unsplit
    assert plan("nvfp4", 1, 12288, 3072, facts={(256, 2): 74}) == (128, 128, 1)
    # N = 9600: 75 CTAs of 128 unsplit; 38 x 2 = 76 at 256 is not a quarter
    # more, 38 x 3 = 114 is
    assert plan("nvfp4", 1, 9600, 3072, facts={(256, 2): 74}) == (128, 128, 1)
    assert plan("nvfp4", 1, 9600, 3072, facts={(256, 2): 74, (256, 3): 45}) == (128, 256, 3)


def test_most_sms_then_the_wider_tile_on_a_tie():
    # N = 6144: 256 x 6 would need 24 > 22 clusters of six; 32 x 4 at 192
    # (128 SMs) beats 24 x 5 at 256 (120)
    assert plan("nvfp4", 1, 6144, 3072) == (128, 192, 4)
    # N = 9216: 72 x 2 at 128 (144 SMs); with room for 36 clusters of four,
    # 36 x 4 at 256 ties at 144 SMs and the wider tile wins
    assert plan("nvfp4", 1, 9216, 3072) == (128, 128, 2)
    more = dict(B200)
    more.update({(256, 4): 36})
    assert plan("nvfp4", 1, 9216, 3072, facts=more) == (128, 256, 4)


def test_host_plan_rejects_bad_arguments():
    L = nvq._lib
    t = (ctypes.c_int * 27)()
    out = (ctypes.c_int * 3)()
    args = lambda fmt=0, M=1, N=12288, K=3072, sms=SMS, table=t: L.nvq_gemm_plan_host(  # noqa: E731
        fmt, M, N, K, sms, table, 1, 1, ctypes.byref(out, 0), ctypes.byref(out, 4), ctypes.byref(out, 8))
    assert args() == 0
    assert args(fmt=4) == -7
    assert args(table=None) == -1
    assert args(sms=0) == -2
    assert args(M=0) == -2
    assert args(N=12) == -2
    assert args(K=128) == -2
