"""GPU parity of the depthwise conv1d (forward, data gradient, weight/bias gradients) against
the fp64 CPU oracle, element by element, through the C ABI.

Workloads: the fp32 parity case (1x200x256, K=9), the conformer forward (16x1500x512, K=9,
bf16), the causal kernel-width sweep (32x750x1024, K in {3,4,5,9,15}, plus C=520, K=7) and
the training-size backward (32x1500x1024, K=9), each at full size and in the launch
configuration the benchmark times, plus small edge cases: T below K, len 0 and T, lengths
outside [0, T], odd C, any K, misaligned buffers (narrow path), guard bands around every
output.

Bars: fp32 I/O max|err| <= 1e-5 * RMS(oracle); bf16 I/O max|err| <= 2e-2 absolute; masked
frames exactly +0.0; dW/dbias (float32 from bf16 inputs) <= 2e-2 absolute and <= 1e-5 * RMS.
"""
import numpy as np
import pytest
import torch

import oracle
import speech_encoder_depthwise_b200 as dw
from gpuhelp import (Guarded, assert_bf16_close, assert_f32_close, assert_masked_zero, dev, max_abs, rms)
from synth import conv1d_inputs, symmetric_pad_left

pytestmark = pytest.mark.gpu

TD = {"bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from speech_encoder_depthwise_b200 import build
    build.build()
    dw.lib()


def gpu_fwd(d, dtype, pad_left, offset=0, bias=True):
    x = dev(d["x"], TD[dtype])
    y = Guarded(x.shape, TD[dtype], offset=offset)
    dw.dwconv1d_fwd(x, dev(d["w"]), dev(d["bias"]) if bias else None, y.t, dev(d["lengths"]), pad_left)
    torch.cuda.synchronize()
    y.check_slack()
    return y.numpy()


def gpu_dx(d, dtype, pad_left, offset=0):
    g = dev(d["dy"], TD[dtype])
    dx = Guarded(g.shape, TD[dtype], offset=offset)
    dw.dwconv1d_bwd_dx(g, dev(d["w"]), dx.t, dev(d["lengths"]), pad_left)
    torch.cuda.synchronize()
    dx.check_slack()
    return dx.numpy()


def gpu_dw(d, dtype, pad_left, K):
    x = dev(d["x"], TD[dtype])
    g = dev(d["dy"], TD[dtype])
    B, T, C = x.shape
    gw = Guarded((K, C), torch.float32)
    gb = Guarded((C,), torch.float32)
    nws = dw.dwconv1d_bwd_dw_workspace_size(B, T, C, K)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
    dw.dwconv1d_bwd_dw(x, g, gw.t, gb.t, dev(d["lengths"]), pad_left, ws)
    torch.cuda.synchronize()
    gw.check_slack()
    gb.check_slack()
    return gw.numpy(), gb.numpy()


def check(dtype, got, ref):
    if dtype == "f32":
        return assert_f32_close(got, ref)
    return assert_bf16_close(got, ref)


# ------------------------------------------------------------------ full-size workloads
def test_fwd_f32_small_workload():
    d = conv1d_inputs(1, 200, 256, 9, dtype="f32", len_range=None, seed=0)
    ref = oracle.dwconv1d_fwd(d["x"], d["w"], d["bias"], None, 4)
    check("f32", gpu_fwd(d, "f32", 4), ref)


def test_fwd_bf16_conformer_workload():
    d = conv1d_inputs(16, 1500, 512, 9, dtype="bf16", len_range=(750, 1500), seed=1)
    ref = oracle.dwconv1d_fwd(d["x"], d["w"], d["bias"], d["lengths"], 4)
    got = gpu_fwd(d, "bf16", 4)
    check("bf16", got, ref)
    assert_masked_zero(got, d["lengths"], 1500)


def test_bwd_bf16_conformer_workload():
    """The backward legs the benchmark times on the conformer workload's shapes."""
    d = conv1d_inputs(16, 1500, 512, 9, dtype="bf16", len_range=(750, 1500), seed=1, with_dy=True)
    ref = oracle.dwconv1d_bwd_dx(d["dy"], d["w"], d["lengths"], 4)
    got = gpu_dx(d, "bf16", 4)
    check("bf16", got, ref)
    assert_masked_zero(got, d["lengths"], 1500)
    rdw, rdb = oracle.dwconv1d_bwd_dw(d["x"], d["dy"], 9, d["lengths"], 4)
    gdw, gdb = gpu_dw(d, "bf16", 4, 9)
    for got, ref in ((gdw, rdw), (gdb, rdb)):
        e = max_abs(got, ref)
        assert e <= 2e-2 and e <= 1e-5 * rms(ref), (e, rms(ref))


@pytest.mark.parametrize("K", [3, 4, 5, 9, 15])
def test_fwd_bf16_causal_sweep(K):
    d = conv1d_inputs(32, 750, 1024, K, dtype="bf16", len_range=(375, 750), seed=2)
    ref = oracle.dwconv1d_fwd(d["x"], d["w"], d["bias"], d["lengths"], K - 1)
    got = gpu_fwd(d, "bf16", K - 1)
    check("bf16", got, ref)
    assert_masked_zero(got, d["lengths"], 750)


def test_fwd_bf16_causal_odd_channels():
    d = conv1d_inputs(32, 750, 520, 7, dtype="bf16", len_range=(375, 750), seed=2)
    ref = oracle.dwconv1d_fwd(d["x"], d["w"], d["bias"], d["lengths"], 6)
    got = gpu_fwd(d, "bf16", 6)
    check("bf16", got, ref)
    assert_masked_zero(got, d["lengths"], 750)


def test_bwd_bf16_training_workload():
    d = conv1d_inputs(32, 1500, 1024, 9, dtype="bf16", len_range=(750, 1500), seed=4, with_dy=True)
    ref = oracle.dwconv1d_bwd_dx(d["dy"], d["w"], d["lengths"], 4)
    got = gpu_dx(d, "bf16", 4)
    check("bf16", got, ref)
    assert_masked_zero(got, d["lengths"], 1500)
    del got, ref
    rdw, rdb = oracle.dwconv1d_bwd_dw(d["x"], d["dy"], 9, d["lengths"], 4)
    gdw, gdb = gpu_dw(d, "bf16", 4, 9)
    for got, ref in ((gdw, rdw), (gdb, rdb)):
        e = max_abs(got, ref)
        assert e <= 2e-2 and e <= 1e-5 * rms(ref), (e, rms(ref))


# ------------------------------------------------------------------ edge cases
EDGE = []
for dtype in ("f32", "bf16"):
    for K in (1, 2, 3, 6, 9, 15, 31, 33):
        for (B, T, C) in ((1, 1, 1), (3, 5, 3), (2, 37, 130), (2, 300, 8), (1, 64, 520)):
            EDGE.append((dtype, K, B, T, C))


@pytest.mark.parametrize("dtype,K,B,T,C", EDGE)
def test_edge_cases_fwd_dx_dw(dtype, K, B, T, C):
    rng = np.random.default_rng(K * 1000 + T * 10 + C)
    d = conv1d_inputs(B, T, C, K, dtype=dtype, len_range=(0, T), seed=int(rng.integers(1 << 30)),
                      with_dy=True)
    if B >= 2:
        d["lengths"][0] = T
        d["lengths"][1] = 0 if T > 4 else d["lengths"][1]
    for pl in sorted({symmetric_pad_left(K), K - 1, 0}):
        ref = oracle.dwconv1d_fwd(d["x"], d["w"], d["bias"], d["lengths"], pl)
        got = gpu_fwd(d, dtype, pl)
        check(dtype, got, ref)
        assert_masked_zero(got, d["lengths"], T)
        ref = oracle.dwconv1d_bwd_dx(d["dy"], d["w"], d["lengths"], pl)
        got = gpu_dx(d, dtype, pl)
        check(dtype, got, ref)
        assert_masked_zero(got, d["lengths"], T)
        rdw, rdb = oracle.dwconv1d_bwd_dw(d["x"], d["dy"], K, d["lengths"], pl)
        gdw, gdb = gpu_dw(d, dtype, pl, K)
        for g, r in ((gdw, rdw), (gdb, rdb)):
            e = max_abs(g, r)
            assert e <= 2e-2 and e <= 1e-5 * max(rms(r), 1e-6), (e, rms(r))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_misaligned_buffers_take_the_narrow_path(dtype):
    d = conv1d_inputs(2, 50, 64, 9, dtype=dtype, len_range=(20, 50), seed=7, with_dy=True)
    ref = oracle.dwconv1d_fwd(d["x"], d["w"], d["bias"], d["lengths"], 4)
    check(dtype, gpu_fwd(d, dtype, 4, offset=1), ref)
    ref = oracle.dwconv1d_bwd_dx(d["dy"], d["w"], d["lengths"], 4)
    check(dtype, gpu_dx(d, dtype, 4, offset=1), ref)


def test_lengths_are_clamped():
    d = conv1d_inputs(3, 40, 16, 5, dtype="bf16", len_range=(0, 40), seed=8)
    d2 = dict(d)
    d["lengths"] = np.array([99, -5, 40], np.int32)
    d2["lengths"] = np.array([40, 0, 40], np.int32)
    a = gpu_fwd(d, "bf16", 2)
    b = gpu_fwd(d2, "bf16", 2)
    np.testing.assert_array_equal(a, b)


def test_no_bias_and_no_lengths():
    d = conv1d_inputs(2, 77, 48, 9, dtype="f32", len_range=None, seed=9)
    ref = oracle.dwconv1d_fwd(d["x"], d["w"], None, None, 4)
    check("f32", gpu_fwd(d, "f32", 4, bias=False), ref)


@pytest.mark.parametrize("K,pl", [(9, 4), (4, 1), (15, 14)])
def test_impulse_is_exact(K, pl):
    """An impulse reproduces the weights exactly (1.0 * w + 0 is exact), reversed along t."""
    T, C, t0 = 64, 32, 30
    w = conv1d_inputs(1, 1, C, K, dtype="bf16", seed=K)["w"]
    x = np.zeros((1, T, C), np.float32)
    x[0, t0] = 1.0
    d = {"x": x, "w": w, "bias": np.zeros(C, np.float32), "lengths": None}
    got = gpu_fwd(d, "bf16", pl)
    expect = np.zeros((T, C))
    for k in range(K):
        expect[t0 + pl - k] = w[k]
    np.testing.assert_array_equal(got[0], expect)
    d["dy"] = x
    got = gpu_dx(d, "bf16", pl)
    expect = np.zeros((T, C))
    for k in range(K):
        expect[t0 - pl + k] = w[k]
    np.testing.assert_array_equal(got[0], expect)


def test_results_are_bitwise_reproducible():
    d = conv1d_inputs(8, 700, 256, 9, dtype="bf16", len_range=(300, 700), seed=11, with_dy=True)
    a = gpu_dw(d, "bf16", 4, 9)
    b = gpu_dw(d, "bf16", 4, 9)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    np.testing.assert_array_equal(gpu_fwd(d, "bf16", 4), gpu_fwd(d, "bf16", 4))


def test_causal_output_ignores_future_frames():
    d = conv1d_inputs(2, 120, 64, 9, dtype="bf16", len_range=None, seed=12)
    base = gpu_fwd(d, "bf16", 8)
    d2 = dict(d)
    x2 = d["x"].copy()
    x2[:, 61:] = 3.0
    d2["x"] = x2
    np.testing.assert_array_equal(gpu_fwd(d2, "bf16", 8)[:, :61], base[:, :61])


@pytest.mark.parametrize("K", [3, 9, 15])
def test_pipelined_and_register_paths_agree(K):
    """16-byte-aligned rows take the bulk-copy pipeline; an input 4 bytes off alignment takes
    the register-tiled kernel.  Both sum the taps in the same order: identical bits."""
    d = conv1d_inputs(3, 300, 256, K, dtype="bf16", len_range=(100, 300), seed=20 + K, with_dy=True)
    x = dev(d["x"], torch.bfloat16)
    raw = torch.empty(x.numel() + 8, dtype=torch.bfloat16, device="cuda")
    xo = raw[2:2 + x.numel()].view(x.shape)
    xo.copy_(x)
    w, bias, ln = dev(d["w"]), dev(d["bias"]), dev(d["lengths"])
    for fn, args in ((dw.dwconv1d_fwd, (w, bias)), (dw.dwconv1d_bwd_dx, (w,))):
        ya, yb = torch.empty_like(x), torch.empty_like(x)
        fn(x, *args, ya, ln, K - 1)
        fn(xo, *args, yb, ln, K - 1)
        torch.cuda.synchronize()
        assert torch.equal(ya.view(torch.int16), yb.view(torch.int16))
    # dW: the two paths add partial sums in different orders; both must meet the bar
    ref = oracle.dwconv1d_bwd_dw(d["x"], d["dy"], K, d["lengths"], K - 1)
    g = dev(d["dy"], torch.bfloat16)
    go = raw.clone()[2:2 + x.numel()].view(x.shape)
    go.copy_(g)
    for xx, gg in ((x, g), (xo, go)):
        gw = torch.empty(K, 256, device="cuda")
        gb = torch.empty(256, device="cuda")
        ws = torch.empty(dw.dwconv1d_bwd_dw_workspace_size(3, 300, 256, K), dtype=torch.uint8, device="cuda")
        dw.dwconv1d_bwd_dw(xx, gg, gw, gb, ln, K - 1, ws)
        torch.cuda.synchronize()
        for got, r in ((gw.cpu().numpy(), ref[0]), (gb.cpu().numpy(), ref[1])):
            e = max_abs(got, r)
            assert e <= 1e-5 * rms(r), (e, rms(r))
