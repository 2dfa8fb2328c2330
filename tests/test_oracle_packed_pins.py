"""Pins of the oracle's packed-batch conv1d (forward, data and weight gradients): sequences back to back
in [N, C], each convolved on its own ("GPU inference for speech", section "Where the time goes":
packed sequences instead of padding).

Pinned against torch float64 conv1d (groups=C) run sequence by sequence with explicit zero
padding, and against the padded-batch oracle with lengths = the sequence lengths (equal on the
valid frames), over lengths including 0 and below K, several K and both padding modes.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import symmetric_pad_left


def torch_seq(x, w, bias, pad_left):
    """One sequence [L, C] through torch's depthwise conv1d, zero-padded pad_left | K-1-pad_left."""
    L, C = x.shape
    K = w.shape[0]
    xt = torch.from_numpy(np.asarray(x, np.float64).T[None])            # [1, C, L]
    xt = torch.nn.functional.pad(xt, (pad_left, K - 1 - pad_left))
    wt = torch.from_numpy(np.asarray(w, np.float64).T[:, None, :])      # [C, 1, K]
    bt = torch.from_numpy(np.asarray(bias, np.float64)) if bias is not None else None
    return torch.nn.functional.conv1d(xt, wt, bt, groups=C)[0].T.numpy()


def torch_seq_dx(dy, w, pad_left):
    L, C = dy.shape
    K = w.shape[0]
    x = torch.zeros(1, C, L, dtype=torch.float64, requires_grad=True)
    wt = torch.from_numpy(np.asarray(w, np.float64).T[:, None, :])
    y = torch.nn.functional.conv1d(torch.nn.functional.pad(x, (pad_left, K - 1 - pad_left)), wt, groups=C)
    y.backward(torch.from_numpy(np.asarray(dy, np.float64).T[None]))
    return x.grad[0].T.numpy()


def torch_seq_dw(x, dy, K, pad_left):
    L, C = x.shape
    w = torch.zeros(C, 1, K, dtype=torch.float64, requires_grad=True)
    b = torch.zeros(C, dtype=torch.float64, requires_grad=True)
    xt = torch.nn.functional.pad(torch.from_numpy(np.asarray(x, np.float64).T[None]), (pad_left, K - 1 - pad_left))
    y = torch.nn.functional.conv1d(xt, w, b, groups=C)
    y.backward(torch.from_numpy(np.asarray(dy, np.float64).T[None]))
    return w.grad[:, 0, :].T.numpy(), b.grad.numpy()


CASES = [(K, mode, seed) for K in (1, 2, 4, 9, 15) for mode in ("sym", "causal") for seed in (0, 1)]


@pytest.mark.parametrize("K,mode,seed", CASES)
def test_packed_matches_torch_per_sequence(K, mode, seed):
    rng = np.random.default_rng(100 * K + seed)
    B, C = int(rng.integers(1, 6)), int(rng.choice([1, 3, 8]))
    lens = rng.integers(0, 40, size=B)
    lens[0] = max(int(lens[0]), 1)
    if B > 2:
        lens[1] = min(K - 1, 2)             # shorter than the window
        lens[2] = 0                         # an empty sequence
    offsets = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    N = int(offsets[-1])
    x = rng.standard_normal((N, C))
    dy = rng.standard_normal((N, C))
    w = rng.standard_normal((K, C))
    bias = rng.standard_normal(C)
    pl = K - 1 if mode == "causal" else symmetric_pad_left(K)
    y = oracle.dwconv1d_fwd_packed(x, w, bias, offsets, pl)
    dx = oracle.dwconv1d_bwd_dx_packed(dy, w, offsets, pl)
    for b in range(B):
        s0, e = offsets[b], offsets[b + 1]
        if e == s0:
            continue
        np.testing.assert_allclose(y[s0:e], torch_seq(x[s0:e], w, bias, pl), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dx[s0:e], torch_seq_dx(dy[s0:e], w, pl), rtol=1e-12, atol=1e-12)
    assert not np.isnan(y).any() and not np.isnan(dx).any()  # every row belongs to a sequence
    gw, gb = oracle.dwconv1d_bwd_dw_packed(x, dy, K, offsets, pl)
    tw, tb = np.zeros((K, C)), np.zeros(C)
    for b in range(B):
        s0, e = offsets[b], offsets[b + 1]
        if e > s0:
            w_b, b_b = torch_seq_dw(x[s0:e], dy[s0:e], K, pl)
            tw += w_b
            tb += b_b
    np.testing.assert_allclose(gw, tw, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(gb, tb, rtol=1e-11, atol=1e-11)


def test_packed_equals_padded_batch_on_valid_frames():
    rng = np.random.default_rng(7)
    B, T, C, K = 4, 30, 5, 9
    lens = np.array([30, 11, 0, 3], dtype=np.int32)
    xp = rng.standard_normal((B, T, C))
    w = rng.standard_normal((K, C))
    bias = rng.standard_normal(C)
    offsets = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    x = np.concatenate([xp[b, :lens[b]] for b in range(B)])
    for pl in (4, 8, 0):
        y = oracle.dwconv1d_fwd_packed(x, w, bias, offsets, pl)
        yp = oracle.dwconv1d_fwd(xp, w, bias, lens, pl)
        for b in range(B):
            np.testing.assert_array_equal(y[offsets[b]:offsets[b + 1]], yp[b, :lens[b]])


def test_uncovered_rows_are_marked():
    x = np.ones((6, 2))
    y = oracle.dwconv1d_fwd_packed(x, np.ones((3, 2)), None, np.array([0, 2, 4], np.int32), 1)
    assert np.isnan(y[4:]).all() and not np.isnan(y[:4]).any()
