"""Pins of the oracle's general depthwise conv2d (forward, data gradient, weight/bias gradients)
against float64 torch conv2d (groups=C) with the same length masks and autograd, over kernel
sizes, strides and symmetric / causal / zero paddings, T from 1, len 0 and T.  The operation is
the NeMo PR's second fused kernel ("Use Fused Kernels for Depthwise Striding Subsampler", section
"What does this PR do ?"): a depthwise conv with fused pre/post masking and causal padding.
"""
import numpy as np
import pytest

import oracle
from pinlib import conv2d_checks

CASES = []
for (KT, KF) in ((3, 3), (1, 1), (2, 3), (5, 1), (3, 5)):
    for stride in ((1, 1), (2, 2), (2, 1), (1, 2)):
        for pads in (((KT - 1) // 2, KT - 1 - (KT - 1) // 2, (KF - 1) // 2), (KT - 1, 0, (KF - 1) // 2), (0, 0, 0)):
            CASES.append((KT, KF, stride, pads))


@pytest.mark.parametrize("KT,KF,stride,pads", CASES)
def test_conv2d_matches_torch_autograd(KT, KF, stride, pads):
    rng = np.random.default_rng(KT * 100 + KF * 10 + stride[0] + 3 * stride[1] + sum(pads))
    for (B, T, F, C) in ((3, 9, 7, 3), (1, 1, 5, 2), (2, 16, 12, 4)):
        fails = conv2d_checks(oracle.default(), rng, B, T, F, C, KT, KF, stride, pads)
        assert not fails, fails


def test_conv2d_equals_the_subsamplers_conv_dw1():
    """With a 3x3 stride-2 window, pads 1|1 (or 2|0) and 1|1, the conv2d is the subsampler's
    conv_dw1 stage: feeding it the h the subsampler builds (one-hot conv0 taps make h = ReLU of
    the shifted mel) reproduces the subsampler's output."""
    rng = np.random.default_rng(11)
    B, T, F, C = 2, 21, 10, 3
    mel = rng.standard_normal((B, T, F)); w1 = rng.standard_normal((3, 3, C)); b1 = rng.standard_normal(C)
    w0 = np.zeros((3, 3, C)); w0[1, 1, :] = 1.0; b0 = np.zeros(C)   # h[i,j] = ReLU(melpad centre tap)
    L = np.array([21, 9], np.int32)
    for causal in (False, True):
        out, ol = oracle.dw_subsample_fwd(mel, w0, b0, w1, b1, L, causal)
        Pt = 2 if causal else 1
        T2, F2 = (T + 1) // 2, (F + 1) // 2
        h = np.zeros((B, T2, F2, C))
        L2 = (L + 1) // 2
        for b in range(B):
            for i in range(min(T2, L2[b])):
                for j in range(F2):
                    t, f = 2 * i + 1 - Pt, 2 * j
                    v = mel[b, t, f] if 0 <= t < L[b] and f < F else 0.0
                    h[b, i, j, :] = max(v, 0.0)
        y, yl = oracle.dwconv2d_fwd(h, w1, b1, L2, (2, 2), (Pt, 2 - Pt, 1))
        assert np.array_equal(yl, ol)
        assert np.max(np.abs(y - out)) <= 1e-12
