"""Pins of the CPU oracle against things other than itself.

* hand-worked golden values (tests/golden/*.json, each citing the definition it follows);
* a second formulation: explicit im2col + matmul, and a dense band matrix for the data
  gradient (brute force on tiny inputs: B in {1,3}, T from 1 (below K) to 50, K in
  {1,2,3,4,5,7,9,15}, C in {1,3,8,9,130}, symmetric and causal, lengths including 0 and T);
* torch's float64 CPU conv1d/conv2d with autograd (a library special case);
* invariants: impulse responses, linearity, exact zeros at masked frames, causality,
  the adjoint identity between forward and data gradient, the exact finite difference of
  the weight gradient, dbias as the sum of the masked dy, the all-ones interior value,
  and the subsampler's closed forms for one-hot kernels.
"""
import numpy as np
import pytest

import oracle
from pinlib import (band_dx, im2col_dw, im2col_fwd, load_golden, pin_battery, rel_err,
                    torch_conv1d_all, torch_subsample)
from synth import conv1d_inputs, subsample_inputs, symmetric_pad_left


def _case(rng, B, T, C, K):
    x = rng.standard_normal((B, T, C))
    w = rng.standard_normal((K, C))
    bias = rng.standard_normal(C)
    dy = rng.standard_normal((B, T, C))
    L = rng.integers(0, T + 1, size=B).astype(np.int32)
    if B >= 2:
        L[0] = T
        L[-1] = 0 if T > 3 else L[-1]
    return x, w, bias, dy, L


# ------------------------------------------------------------------ golden values
def test_golden_conv1d_worked_example():
    g = load_golden("dwconv1d_worked_example.json")
    x = np.array(g["x"], float); w = np.array(g["w"], float); bias = np.array(g["bias"], float)
    dy = np.array(g["dy"], float); L = np.array(g["lengths"], np.int32)
    s = g["symmetric"]
    np.testing.assert_array_equal(oracle.dwconv1d_fwd(x, w, bias, L, s["pad_left"]), s["y"])
    np.testing.assert_array_equal(oracle.dwconv1d_bwd_dx(dy, w, L, s["pad_left"]), s["dx"])
    dw, db = oracle.dwconv1d_bwd_dw(x, dy, 3, L, s["pad_left"])
    np.testing.assert_array_equal(dw, s["dw"])
    np.testing.assert_array_equal(db, s["dbias"])
    c = g["causal_no_bias"]
    np.testing.assert_array_equal(oracle.dwconv1d_fwd(x, w, None, L, c["pad_left"]), c["y"])


@pytest.mark.parametrize("mode,causal", [("symmetric", False), ("causal", True)])
def test_golden_subsample_worked_example(mode, causal):
    g = load_golden("subsample_worked_example.json")
    e = g[mode]
    out, ol = oracle.dw_subsample_fwd(np.array(g["mel"], float), np.array(e["w0"], float),
                                      np.array(e["b0"], float), np.array(g["w1"], float),
                                      np.array(g["b1"], float), np.array(g["lengths"], np.int32),
                                      causal)
    np.testing.assert_array_equal(out, e["out"])
    assert list(ol) == e["out_lengths"]


# ------------------------------------------------------------------ second formulation
@pytest.mark.parametrize("K", [1, 2, 3, 4, 5, 7, 9, 15])
@pytest.mark.parametrize("mode", ["symmetric", "causal"])
def test_conv1d_matches_im2col_bruteforce(K, mode):
    rng = np.random.default_rng(K * 10 + (mode == "causal"))
    pl = symmetric_pad_left(K) if mode == "symmetric" else K - 1
    for B in (1, 3):
        for T in (1, 2, K - 1 if K > 1 else 1, K, K + 1, 17, 50):
            for C in (1, 3, 8, 9, 130):
                if C == 130 and T not in (K, 50):
                    continue
                x, w, bias, dy, L = _case(rng, B, T, C, K)
                y = oracle.dwconv1d_fwd(x, w, bias, L, pl)
                assert rel_err(y, im2col_fwd(x, w, bias, L, pl)) <= 1e-12
                dx = oracle.dwconv1d_bwd_dx(dy, w, L, pl)
                if T <= 50 and C <= 9:
                    assert rel_err(dx, band_dx(dy, w, L, pl)) <= 1e-12
                dw, db = oracle.dwconv1d_bwd_dw(x, dy, K, L, pl)
                rdw, rdb = im2col_dw(x, dy, K, L, pl)
                assert rel_err(dw, rdw) <= 1e-12
                assert rel_err(db, rdb) <= 1e-12


@pytest.mark.parametrize("B,T,C,K,pl", [(2, 64, 24, 9, 4), (3, 40, 17, 15, 14), (1, 33, 130, 7, 3),
                                        (4, 25, 8, 4, 1), (2, 3, 5, 9, 4)])
def test_conv1d_matches_torch_autograd(B, T, C, K, pl):
    rng = np.random.default_rng(B * 1000 + T)
    x, w, bias, dy, L = _case(rng, B, T, C, K)
    ty, tdx, tdw, tdb = torch_conv1d_all(x, w, bias, dy, L, pl)
    assert rel_err(oracle.dwconv1d_fwd(x, w, bias, L, pl), ty) <= 1e-12
    assert rel_err(oracle.dwconv1d_bwd_dx(dy, w, L, pl), tdx) <= 1e-12
    dw, db = oracle.dwconv1d_bwd_dw(x, dy, K, L, pl)
    assert rel_err(dw, tdw) <= 1e-12
    assert rel_err(db, tdb) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,T,F,C", [(1, 1, 1, 1), (2, 9, 7, 3), (3, 30, 16, 5), (2, 64, 80, 4)])
def test_subsample_matches_torch(causal, B, T, F, C):
    rng = np.random.default_rng(T * 7 + F)
    mel = rng.standard_normal((B, T, F))
    w0 = rng.standard_normal((3, 3, C)); w1 = rng.standard_normal((3, 3, C))
    b0 = rng.standard_normal(C); b1 = rng.standard_normal(C)
    L = rng.integers(0, T + 1, size=B).astype(np.int32)
    L[0] = T
    out, ol = oracle.dw_subsample_fwd(mel, w0, b0, w1, b1, L, causal)
    ref, rl = torch_subsample(mel, w0, b0, w1, b1, L, causal)
    assert out.shape == ref.shape
    assert rel_err(out, ref) <= 1e-12
    np.testing.assert_array_equal(ol, rl)


# ------------------------------------------------------------------ invariants
@pytest.mark.parametrize("K,pl", [(9, 4), (4, 1), (5, 4), (1, 0), (15, 14)])
def test_impulse_identities(K, pl):
    """A forward impulse at t0 reads w backwards along t; a backward impulse reads w as stored."""
    T, C, t0 = 40, 3, 20
    rng = np.random.default_rng(K)
    w = rng.standard_normal((K, C))
    x = np.zeros((1, T, C)); x[0, t0, :] = 1.0
    y = oracle.dwconv1d_fwd(x, w, None, None, pl)
    expect = np.zeros((T, C))
    for k in range(K):
        expect[t0 + pl - k] = w[k]
    np.testing.assert_array_equal(y[0], expect)
    dy = np.zeros((1, T, C)); dy[0, t0, :] = 1.0
    dx = oracle.dwconv1d_bwd_dx(dy, w, None, pl)
    expect = np.zeros((T, C))
    for k in range(K):
        expect[t0 - pl + k] = w[k]
    np.testing.assert_array_equal(dx[0], expect)


def test_linearity():
    rng = np.random.default_rng(5)
    B, T, C, K, pl = 2, 37, 6, 9, 4
    x1 = rng.standard_normal((B, T, C)); x2 = rng.standard_normal((B, T, C))
    w = rng.standard_normal((K, C)); bias = rng.standard_normal(C)
    L = np.array([30, 37], np.int32)
    a, b = 0.75, -1.5
    f = lambda x: oracle.dwconv1d_fwd(x, w, bias, L, pl)
    mask = (np.arange(T)[None, :] < L[:, None])[:, :, None]
    lhs = f(a * x1 + b * x2) - bias * mask
    rhs = a * (f(x1) - bias * mask) + b * (f(x2) - bias * mask)
    assert np.max(np.abs(lhs - rhs)) <= 1e-12 * np.max(np.abs(rhs))


def test_masked_frames_exact_zero():
    rng = np.random.default_rng(6)
    B, T, C, K = 3, 25, 4, 9
    x = rng.standard_normal((B, T, C)) + 10.0
    w = rng.standard_normal((K, C)); bias = rng.standard_normal(C) + 3.0
    dy = rng.standard_normal((B, T, C)) + 10.0
    L = np.array([0, 7, 25], np.int32)
    y = oracle.dwconv1d_fwd(x, w, bias, L, 4)
    dx = oracle.dwconv1d_bwd_dx(dy, w, L, 4)
    for b in range(B):
        for arr in (y, dx):
            tail = arr[b, L[b]:]
            assert np.all(tail == 0.0) and not np.any(np.signbit(tail))
    # values at and beyond len never reach the valid outputs
    x2 = x.copy(); x2[1, 7:] = -99.0
    np.testing.assert_array_equal(oracle.dwconv1d_fwd(x2, w, bias, L, 4), y)
    dy2 = dy.copy(); dy2[1, 7:] = 55.0
    np.testing.assert_array_equal(oracle.dwconv1d_bwd_dx(dy2, w, L, 4), dx)
    dw, db = oracle.dwconv1d_bwd_dw(x, dy, K, L, 4)
    dw2, db2 = oracle.dwconv1d_bwd_dw(x2, dy2, K, L, 4)
    np.testing.assert_array_equal(dw, dw2)
    np.testing.assert_array_equal(db, db2)


@pytest.mark.parametrize("K", [3, 4, 9, 15])
def test_causal_outputs_ignore_future(K):
    rng = np.random.default_rng(K + 100)
    T, C = 30, 5
    x = rng.standard_normal((2, T, C)); w = rng.standard_normal((K, C)); bias = rng.standard_normal(C)
    y = oracle.dwconv1d_fwd(x, w, bias, None, K - 1)
    for t in (0, 9, 17, 28):
        x2 = x.copy(); x2[:, t + 1:] = rng.standard_normal((2, T - t - 1, C))
        y2 = oracle.dwconv1d_fwd(x2, w, bias, None, K - 1)
        np.testing.assert_array_equal(y2[:, :t + 1], y[:, :t + 1])


@pytest.mark.parametrize("K,pl", [(9, 4), (4, 3), (7, 3), (2, 0)])
def test_adjoint_identity(K, pl):
    """<dy, fwd_nobias(x)> = <bwd_dx(dy), x>."""
    rng = np.random.default_rng(K * 3 + pl)
    B, T, C = 3, 41, 7
    x = rng.standard_normal((B, T, C)); dy = rng.standard_normal((B, T, C))
    w = rng.standard_normal((K, C)); L = np.array([41, 20, 3], np.int32)
    lhs = np.sum(dy * oracle.dwconv1d_fwd(x, w, None, L, pl))
    rhs = np.sum(oracle.dwconv1d_bwd_dx(dy, w, L, pl) * x)
    assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(lhs))


def test_dw_finite_difference_exact():
    """<dy, y> is linear in w, so its difference under w + e_kc is exactly dW[k,c]."""
    rng = np.random.default_rng(9)
    B, T, C, K, pl = 2, 23, 4, 5, 2
    x = rng.standard_normal((B, T, C)); dy = rng.standard_normal((B, T, C))
    w = rng.standard_normal((K, C)); bias = rng.standard_normal(C)
    L = np.array([23, 11], np.int32)
    dw, db = oracle.dwconv1d_bwd_dw(x, dy, K, L, pl)
    base = np.sum(dy * oracle.dwconv1d_fwd(x, w, bias, L, pl))
    for k in range(K):
        for c in range(C):
            w2 = w.copy(); w2[k, c] += 1.0
            d = np.sum(dy * oracle.dwconv1d_fwd(x, w2, bias, L, pl)) - base
            assert abs(d - dw[k, c]) <= 1e-9 * max(1.0, abs(dw[k, c]))
    for c in range(C):
        b2 = bias.copy(); b2[c] += 1.0
        d = np.sum(dy * oracle.dwconv1d_fwd(x, w, b2, L, pl)) - base
        assert abs(d - db[c]) <= 1e-9 * max(1.0, abs(db[c]))


def test_dbias_is_sum_of_masked_dy():
    rng = np.random.default_rng(10)
    B, T, C, K = 3, 19, 6, 3
    x = rng.standard_normal((B, T, C)); dy = rng.standard_normal((B, T, C))
    L = np.array([19, 4, 0], np.int32)
    _, db = oracle.dwconv1d_bwd_dw(x, dy, K, L, 1)
    expect = dy[0].sum(0) + dy[1, :4].sum(0)
    assert np.max(np.abs(db - expect)) <= 1e-12 * np.max(np.abs(expect))


def test_all_ones_interior():
    rng = np.random.default_rng(11)
    T, C, K, pl = 30, 5, 9, 4
    w = rng.standard_normal((K, C)); bias = rng.standard_normal(C)
    y = oracle.dwconv1d_fwd(np.ones((1, T, C)), w, bias, None, pl)
    interior = y[0, pl:T - (K - 1 - pl)]
    assert np.max(np.abs(interior - (bias + w.sum(0)))) <= 1e-12


def test_edge_cases():
    w = np.ones((9, 3))
    assert oracle.dwconv1d_fwd(np.zeros((0, 5, 3)), w, None, None, 4).shape == (0, 5, 3)
    assert oracle.dwconv1d_fwd(np.zeros((2, 0, 3)), w, None, None, 4).shape == (2, 0, 3)
    # T < K: only the real frames enter the sum
    x = np.array([[[1.0, 2.0, 3.0], [4.0, 5.0, 6.0]]])
    y = oracle.dwconv1d_fwd(x, w, None, None, 4)
    np.testing.assert_array_equal(y[0], [[5.0, 7.0, 9.0], [5.0, 7.0, 9.0]])
    # lengths outside [0, T] are clamped
    x = np.random.default_rng(0).standard_normal((2, 6, 3))
    a = oracle.dwconv1d_fwd(x, w, None, np.array([99, -4], np.int32), 4)
    b = oracle.dwconv1d_fwd(x, w, None, np.array([6, 0], np.int32), 4)
    np.testing.assert_array_equal(a, b)
    with pytest.raises(ValueError):
        oracle.dwconv1d_fwd(x, w, None, None, 9)


# ------------------------------------------------------------------ subsampler closed forms
@pytest.mark.parametrize("causal", [False, True])
def test_subsample_onehot_closed_form(causal):
    """With one-hot kernels both stages become shifted copies: out = w1c * ReLU(b0 + w0c * mel[r, f])."""
    rng = np.random.default_rng(12 + causal)
    B, T, F, C = 2, 21, 10, 3
    mel = rng.standard_normal((B, T, F))
    L = np.array([21, 9], np.int32)
    w0 = np.zeros((3, 3, C)); w1 = np.zeros((3, 3, C))
    p0, q0, p1, q1 = 2, 1, 2, 1      # bottom-centre taps: row 2i + 2 - Pt, column 2j
    w0[p0, q0] = rng.uniform(0.5, 2, C); w1[p1, q1] = rng.uniform(0.5, 2, C)
    b0 = rng.standard_normal(C); b1 = np.zeros(C)
    out, ol = oracle.dw_subsample_fwd(mel, w0, b0, w1, b1, L, causal)
    pt = 2 if causal else 1
    T4, F4 = out.shape[1:3]
    for b in range(B):
        L2 = (L[b] + 1) // 2; L4 = (L2 + 1) // 2
        assert ol[b] == L4
        for i in range(T4):
            for j in range(F4):
                hr, hc = 2 * i + p1 - pt, 2 * j + q1 - 1
                if i >= L4:
                    expect = np.zeros(C)
                elif hr < 0 or hr >= L2 or hc < 0:
                    expect = np.zeros(C)
                else:
                    mr, mc = 2 * hr + p0 - pt, 2 * hc + q0 - 1
                    mv = mel[b, mr, mc] if (0 <= mr < L[b] and 0 <= mc < F) else 0.0
                    expect = w1[p1, q1] * np.maximum(b0 + w0[p0, q0] * mv, 0.0)
                np.testing.assert_allclose(out[b, i, j], expect, rtol=1e-14, atol=0)


@pytest.mark.parametrize("causal", [False, True])
def test_subsample_masking_and_causality(causal):
    d = subsample_inputs(2, 40, 12, 4, len_range=(10, 40), seed=3)
    out, ol = oracle.dw_subsample_fwd(d["mel"], d["w0"], d["b0"], d["w1"], d["b1"], d["lengths"], causal)
    for b in range(2):
        tail = out[b, ol[b]:]
        assert np.all(tail == 0.0) and not np.any(np.signbit(tail))
    if causal:
        # out row i reads h rows <= 2i, which read mel rows <= 4i
        mel2 = d["mel"].copy()
        for i in (0, 3, 6):
            mel2[:, 4 * i + 1:] = 7.0
            o2, _ = oracle.dw_subsample_fwd(mel2, d["w0"], d["b0"], d["w1"], d["b1"],
                                            np.array([40, 40], np.int32), causal)
            o1, _ = oracle.dw_subsample_fwd(d["mel"], d["w0"], d["b0"], d["w1"], d["b1"],
                                            np.array([40, 40], np.int32), causal)
            np.testing.assert_array_equal(o2[:, :i + 1], o1[:, :i + 1])
            mel2 = d["mel"].copy()


def test_generator_recipe():
    d = conv1d_inputs(2, 10, 8, 9, dtype="bf16", len_range=(5, 10), seed=1, with_dy=True)
    for k in ("x", "w", "bias", "dy"):
        u = d[k].view(np.uint32)
        assert np.all((u & 0xFFFF) == 0)
    assert d["lengths"].dtype == np.int32 and np.all((d["lengths"] >= 5) & (d["lengths"] <= 10))
    s = subsample_inputs(2, 20, 8, 4, len_range=(10, 20), seed=3)
    for b in range(2):
        assert np.all(s["mel"][b, s["lengths"][b]:] == 0)


def test_pin_battery_passes_on_the_oracle():
    assert pin_battery(oracle.default()) == []
