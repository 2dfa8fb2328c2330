"""GPU parity at the size limits the ABI accepts, against the fp64 CPU oracle, through the C ABI.

- the largest accepted channel count (C = 2^22) for the conv1d forward, data gradient and weight
  gradient (32768 channel tiles: more tiles than resident blocks);
- a long sequence (T = 2^20 frames) for the conv1d forward and weight gradient;
- the subsampler with more items (4097) than its balanced unit deal handles (round robin);
- the conv2d kernels with 65536 channels (1024 channel slabs);
- the widest accepted kernel (K = 4096, longer than the sequence) and 4096 streams of the
  streaming conv.
Bars as in the other parity tests (bf16: <= max(2e-2, 1 ulp) and faithful; weight gradients
<= 2e-2 absolute and <= 1e-5 * RMS).
"""
import numpy as np
import pytest
import torch

import oracle
import speech_encoder_depthwise_b200 as dw
from gpuhelp import Guarded, assert_bf16_close, dev, max_abs, rms
from synth import conv1d_inputs, conv2d_inputs, subsample_inputs

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from speech_encoder_depthwise_b200 import build
    build.build()
    dw.lib()


def grads_close(got, ref):
    for g, r in zip(got, ref):
        e = max_abs(g, r)
        assert e <= 2e-2 and e <= 1e-5 * max(rms(r), 1e-6), (e, rms(r))


def conv1d_all(d, K, pl):
    B, T, C = d["x"].shape
    x, g, w = dev(d["x"], BF), dev(d["dy"], BF), dev(d["w"])
    ln = dev(d["lengths"])
    y = Guarded((B, T, C), BF)
    dw.dwconv1d_fwd(x, w, dev(d["bias"]), y.t, ln, pl)
    dx = Guarded((B, T, C), BF)
    dw.dwconv1d_bwd_dx(g, w, dx.t, ln, pl)
    gw, gb = Guarded((K, C), torch.float32), Guarded((C,), torch.float32)
    ws = torch.empty(max(dw.dwconv1d_bwd_dw_workspace_size(B, T, C, K), 16), dtype=torch.uint8, device="cuda")
    dw.dwconv1d_bwd_dw(x, g, gw.t, gb.t, ln, pl, ws)
    torch.cuda.synchronize()
    for o in (y, dx, gw, gb):
        o.check_slack()
    assert_bf16_close(y.numpy(), oracle.dwconv1d_fwd(d["x"], d["w"], d["bias"], d["lengths"], pl))
    assert_bf16_close(dx.numpy(), oracle.dwconv1d_bwd_dx(d["dy"], d["w"], d["lengths"], pl))
    grads_close((gw.numpy(), gb.numpy()), oracle.dwconv1d_bwd_dw(d["x"], d["dy"], K, d["lengths"], pl))


def test_largest_channel_count():
    d = conv1d_inputs(1, 5, 1 << 22, 3, dtype="bf16", len_range=(4, 4), seed=1, with_dy=True)
    conv1d_all(d, 3, 1)


def test_long_sequence():
    d = conv1d_inputs(1, 1 << 20, 16, 9, dtype="bf16", len_range=((1 << 20) - 1000, (1 << 20) - 1000), seed=2,
                      with_dy=True)
    conv1d_all(d, 9, 4)


def test_subsampler_more_items_than_the_balanced_deal():
    B, T, F, C = 4097, 8, 8, 32
    s = subsample_inputs(B, T, F, C, len_range=(0, T), seed=4)
    T4, F4 = dw.subsample_out_shape(T, F)
    out = Guarded((B, T4, F4, C), BF)
    ol = torch.empty(B, dtype=torch.int32, device="cuda")
    dw.dw_subsample_fwd(dev(s["mel"]), dev(s["w0"]), dev(s["b0"]), dev(s["w1"]), dev(s["b1"]), out.t,
                        dev(s["lengths"]), ol, 0)
    torch.cuda.synchronize()
    out.check_slack()
    ref, rl = oracle.dw_subsample_fwd(s["mel"], s["w0"], s["b0"], s["w1"], s["b1"], s["lengths"], False)
    assert_bf16_close(out.numpy(), ref)
    assert np.array_equal(ol.cpu().numpy(), rl)


def test_conv2d_many_channel_slabs():
    B, T, F, C = 1, 9, 5, 1 << 16
    stride, pads = (2, 2), (1, 1, 1)
    To, Fo = dw.conv2d_out_shape(T, F, 3, 3, stride, pads)
    d = conv2d_inputs(B, T, F, C, 3, 3, dtype="bf16", len_range=(7, 7), seed=3, dy_shape=(B, To, Fo, C))
    x, g, w = dev(d["x"], BF), dev(d["dy"], BF), dev(d["w"])
    ln = dev(d["lengths"])
    y = Guarded((B, To, Fo, C), BF)
    dw.dwconv2d_fwd(x, w, dev(d["bias"]), y.t, ln, None, stride, pads)
    dx = Guarded((B, T, F, C), BF)
    dw.dwconv2d_bwd_dx(g, w, dx.t, ln, stride, pads)
    gw, gb = Guarded((3, 3, C), torch.float32), Guarded((C,), torch.float32)
    ws = torch.empty(dw.dwconv2d_bwd_dw_workspace_size(B, T, F, C, 3, 3, stride, pads), dtype=torch.uint8,
                     device="cuda")
    dw.dwconv2d_bwd_dw(x, g, gw.t, gb.t, ln, stride, pads, ws)
    torch.cuda.synchronize()
    for o in (y, dx, gw, gb):
        o.check_slack()
    assert_bf16_close(y.numpy(), oracle.dwconv2d_fwd(d["x"], d["w"], d["bias"], d["lengths"], stride, pads)[0])
    assert_bf16_close(dx.numpy(), oracle.dwconv2d_bwd_dx(d["dy"], d["w"], d["lengths"], T, F, stride, pads))
    grads_close((gw.numpy(), gb.numpy()), oracle.dwconv2d_bwd_dw(d["x"], d["dy"], 3, 3, d["lengths"], stride, pads))


def test_widest_kernel():
    """K = 4096 (the largest accepted width), far longer than the sequence: the runtime-width
    kernels and the weight gradient's passes of taps."""
    d = conv1d_inputs(2, 100, 8, 4096, dtype="bf16", len_range=(60, 100), seed=6, with_dy=True)
    conv1d_all(d, 4096, 2048)


def test_many_streams():
    B, T, C, K = 4096, 1, 64, 9
    rng = np.random.default_rng(8)
    from synth import bf16_round
    w = bf16_round(rng.standard_normal((K, C)) / 3.0)
    b = bf16_round(rng.standard_normal(C) * 0.3)
    cache = torch.zeros(B, K - 1, C, dtype=BF, device="cuda")
    cache_o = np.zeros((B, K - 1, C))
    for _ in range(3):
        x = bf16_round(rng.standard_normal((B, T, C)))
        y = torch.empty(B, T, C, dtype=BF, device="cuda")
        dw.dwconv1d_stream_fwd(dev(x, BF), dev(w), dev(b), y, cache, None)
        torch.cuda.synchronize()
        ry, cache_o = oracle.dwconv1d_stream_fwd(x, w, b, cache_o, None)
        assert_bf16_close(y.float().cpu().numpy(), ry)
        assert np.array_equal(cache.float().cpu().numpy(), cache_o)
