"""Pins of the oracle's subsampler backward (gradients of sum(out * dout) with respect to w0, b0,
w1, b1) against formulations that are not the oracle's own code: float64 autograd through
torch's conv2d / relu / masks, and exact finite differences of <dout, out> in w1 and b1 (out is
linear in both).  The fused kernels of NeMo PR #16114 ("What does this PR do ?") come with their
backward passes for training; this is their definition.
"""
import numpy as np
import pytest

import oracle
from pinlib import subsample_bwd_checks, torch_subsample_grads, rel_err


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,T,F,C", [(1, 1, 1, 1), (2, 5, 7, 3), (3, 13, 10, 4), (2, 31, 16, 5), (1, 8, 80, 2)])
def test_backward_matches_autograd_and_finite_differences(B, T, F, C, causal):
    rng = np.random.default_rng(B * 1000 + T * 10 + F + C)
    fails = subsample_bwd_checks(oracle.default(), rng, B, T, F, C, causal)
    assert not fails, fails


def test_zero_dout_gives_zero_gradients_and_len0_items_contribute_nothing():
    rng = np.random.default_rng(3)
    mel = rng.standard_normal((2, 9, 6)); w0 = rng.standard_normal((3, 3, 2)); b0 = rng.standard_normal(2)
    w1 = rng.standard_normal((3, 3, 2))
    T4, F4 = oracle.subsample_out_shape(9, 6, False)
    g = oracle.dw_subsample_bwd(mel, w0, b0, w1, np.zeros((2, T4, F4, 2)), None, False)
    assert all(np.all(a == 0.0) for a in g)
    dout = rng.standard_normal((2, T4, F4, 2))
    both = oracle.dw_subsample_bwd(mel, w0, b0, w1, dout, np.array([9, 0], np.int32), False)
    first = oracle.dw_subsample_bwd(mel[:1], w0, b0, w1, dout[:1], np.array([9], np.int32), False)
    for a, b in zip(both, first):
        assert rel_err(a, b) <= 1e-14


def test_db1_is_the_masked_sum_of_dout():
    rng = np.random.default_rng(4)
    mel = rng.standard_normal((3, 20, 8)); w0 = rng.standard_normal((3, 3, 4)); b0 = rng.standard_normal(4)
    w1 = rng.standard_normal((3, 3, 4)); L = np.array([20, 7, 1], np.int32)
    T4, F4 = oracle.subsample_out_shape(20, 8, True)
    dout = rng.standard_normal((3, T4, F4, 4))
    _, _, _, db1 = oracle.dw_subsample_bwd(mel, w0, b0, w1, dout, L, True)
    L4 = ((L + 1) // 2 + 1) // 2
    expect = sum(dout[b, :L4[b]].sum(axis=(0, 1)) for b in range(3))
    assert rel_err(db1, expect) <= 1e-14
