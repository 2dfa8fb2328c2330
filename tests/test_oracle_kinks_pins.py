"""Pins of the oracle's kink budget for the subsampler backward (oracle_dw_subsample_bwd_kinks).

The ReLU derivative [z > 0] of conv0's output is a decision taken on a floating-point z (NeMo
PR #16114, "What does this PR do ?": conv0 -> ReLU -> masking -> conv_dw1, with its backward for
training).  Where a float32 evaluation of z and the float64 one can disagree on the sign, the
weight gradients dw0 / db0 may move by |dh| |mel tap| / |dh| per such pixel; the budget sums those
bounds.  It is pinned here against a brute-force recount written with torch (unfold patches,
autograd for dh), at thresholds that take no pixel (the budget must be exactly 0), some and all.
"""
import numpy as np
import pytest

import oracle
from pinlib import rel_err, subsample_kink_checks, torch_subsample_kinks


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,T,F,C", [(1, 1, 1, 1), (2, 5, 7, 3), (3, 13, 10, 4), (2, 30, 17, 5), (1, 9, 80, 2)])
def test_kink_budget_matches_brute_force(B, T, F, C, causal):
    rng = np.random.default_rng(B * 100 + T * 7 + F + C)
    assert not subsample_kink_checks(oracle.default(), rng, B, T, F, C, causal)


def test_kink_budget_counts_exact_zeros_only_at_zero_threshold():
    # z = b0 + sum mel w0 with b0 = 0 and a zero mel window: every valid pixel has z == 0 exactly
    B, T, F, C = 1, 6, 4, 2
    mel = np.zeros((B, T, F)); w0 = np.ones((3, 3, C)); b0 = np.zeros(C); w1 = np.ones((3, 3, C))
    T4, F4 = oracle.subsample_out_shape(T, F, False)
    dout = np.ones((B, T4, F4, C))
    kdw0, kdb0 = oracle.dw_subsample_bwd_kinks(mel, w0, b0, w1, dout, np.array([4], np.int32), False, 0.0)
    rdw0, rdb0 = torch_subsample_kinks(mel, w0, b0, w1, dout, np.array([4], np.int32), False, 0.0, 0.0)
    assert np.all(kdw0 == 0.0)            # |mel tap| = 0 everywhere
    assert rel_err(kdb0, rdb0) == 0.0 and np.all(kdb0 > 0.0)


def test_relative_threshold_scales_with_term_magnitudes():
    # scaling every input of z by 2 doubles z and S: the same pixels count
    rng = np.random.default_rng(11)
    mel = rng.standard_normal((2, 12, 9)); w0 = rng.standard_normal((3, 3, 3)) / 3
    b0 = rng.standard_normal(3) * 0.3; w1 = rng.standard_normal((3, 3, 3)) / 3
    L = np.array([12, 7], np.int32)
    T4, F4 = oracle.subsample_out_shape(12, 9, True)
    dout = rng.standard_normal((2, T4, F4, 3))
    a = oracle.dw_subsample_bwd_kinks(mel, w0, b0, w1, dout, L, True, 0.0, 0.25)
    b = oracle.dw_subsample_bwd_kinks(mel, 2 * w0, 2 * b0, w1, dout, L, True, 0.0, 0.25)
    assert rel_err(a[1], b[1]) <= 1e-14 and rel_err(a[0], b[0]) <= 1e-14
    assert np.any(a[1] > 0.0)
