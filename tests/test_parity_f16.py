"""GPU parity of the fp16 I/O variants (dtype DW_F16) of every entry point against the fp64
CPU oracle, element by element, through the C ABI.

fp16 ("GPU inference for speech", section "Precision": 16-bit inference in FP16 or BF16) keeps
float32 weights and float32 arithmetic; only the activations are 16-bit.  Inputs are drawn as
for the other workloads and rounded to fp16 values, so the oracle reads exactly what the GPU
reads.  Bars: outputs faithfully rounded to fp16 (|gpu - oracle| < ulp_f16(oracle) + 1e-5) with
masked frames +0.0; weight gradients (float32) <= 2e-2 absolute and <= 1e-5 * RMS.

Cases: the conformer shape (16x1500x512, K=9, symmetric) for forward, dX, dW and the one-pass
backward; a causal K=15 and a runtime K=6; C that takes 2- and 1-channel vectors; misaligned
buffers (narrow path); the streaming conv over chunks; the conv2d subsampler-stage shape on the
TMA path and windows/strides of the general kernels; the workspace-free dW; the subsampler with
fp16 output (tensor-core kernel and, for an odd C, the SIMT kernel) and its backward with fp16
dout (bars as for bf16 dout: 1e-5 * RMS plus the oracle's ReLU-kink budget).
"""
import numpy as np
import pytest
import torch

import oracle
import speech_encoder_depthwise_b200 as dw
from gpuhelp import Guarded, assert_f16_close, assert_masked_zero, dev, max_abs, rms
from synth import conv1d_inputs, conv2d_inputs, f16_round, subsample_inputs, symmetric_pad_left

pytestmark = pytest.mark.gpu
H = torch.float16


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from speech_encoder_depthwise_b200 import build
    build.build()
    dw.lib()


def grads_close(got, ref):
    for g, r in zip(got, ref):
        e = max_abs(g, r)
        assert e <= 2e-2 and e <= 1e-5 * max(rms(r), 1e-6), (e, rms(r))


def to_dev(a, offset=0):
    g = Guarded(a.shape, H, offset=offset)
    g.t.copy_(torch.from_numpy(np.ascontiguousarray(a)).to(H))
    return g


def run_conv1d(d, K, pad_left, offset=0, bwd=True):
    B, T, C = d["x"].shape
    L = d["lengths"]
    x = to_dev(d["x"], offset)
    y = Guarded((B, T, C), H, offset=offset)
    dw.dwconv1d_fwd(x.t, dev(d["w"]), dev(d["bias"]), y.t, dev(L), pad_left)
    torch.cuda.synchronize()
    y.check_slack()
    got = y.numpy()
    assert_f16_close(got, oracle.dwconv1d_fwd(d["x"], d["w"], d["bias"], L, pad_left))
    assert_masked_zero(got, L, T)
    if not bwd:
        return
    g = to_dev(d["dy"], offset)
    dx = Guarded((B, T, C), H, offset=offset)
    dw.dwconv1d_bwd_dx(g.t, dev(d["w"]), dx.t, dev(L), pad_left)
    torch.cuda.synchronize()
    dx.check_slack()
    rdx = oracle.dwconv1d_bwd_dx(d["dy"], d["w"], L, pad_left)
    assert_f16_close(dx.numpy(), rdx)
    assert_masked_zero(dx.numpy(), L, T)
    rdw = oracle.dwconv1d_bwd_dw(d["x"], d["dy"], K, L, pad_left)
    gw, gb = Guarded((K, C), torch.float32), Guarded((C,), torch.float32)
    ws = torch.empty(max(dw.dwconv1d_bwd_dw_workspace_size(B, T, C, K), 16), dtype=torch.uint8, device="cuda")
    dw.dwconv1d_bwd_dw(x.t, g.t, gw.t, gb.t, dev(L), pad_left, ws)
    torch.cuda.synchronize()
    grads_close((gw.numpy(), gb.numpy()), rdw)
    # the one-pass backward: the same dx and gradients
    dx2 = Guarded((B, T, C), H, offset=offset)
    dw.dwconv1d_bwd(x.t, g.t, dev(d["w"]), dx2.t, gw.t, gb.t, dev(L), pad_left, ws)
    torch.cuda.synchronize()
    dx2.check_slack()
    assert_f16_close(dx2.numpy(), rdx)
    grads_close((gw.numpy(), gb.numpy()), rdw)
    # the workspace-free weight gradient
    dw.dwconv1d_bwd_dw_noalloc(x.t, g.t, gw.t, gb.t, dev(L), pad_left)
    torch.cuda.synchronize()
    grads_close((gw.numpy(), gb.numpy()), rdw)


def test_conformer_workload():
    d = conv1d_inputs(16, 1500, 512, 9, dtype="f16", len_range=(750, 1500), seed=1, with_dy=True)
    run_conv1d(d, 9, 4)


@pytest.mark.parametrize("K,pad", [(15, "causal"), (6, "sym"), (4, "causal"), (1, "sym")])
def test_widths(K, pad):
    d = conv1d_inputs(3, 170, 256, K, dtype="f16", len_range=(0, 170), seed=K, with_dy=True)
    d["lengths"][0] = 170
    run_conv1d(d, K, K - 1 if pad == "causal" else symmetric_pad_left(K))


@pytest.mark.parametrize("C", [130, 7])
def test_narrow_channel_vectors(C):
    d = conv1d_inputs(2, 90, C, 9, dtype="f16", len_range=(10, 90), seed=C, with_dy=True)
    run_conv1d(d, 9, 4)


def test_misaligned_buffers_take_the_narrow_path():
    d = conv1d_inputs(2, 60, 64, 9, dtype="f16", len_range=(20, 60), seed=3, with_dy=True)
    run_conv1d(d, 9, 4, offset=1)


@pytest.mark.parametrize("K", [9, 20])
def test_streaming_chunks(K):
    rng = np.random.default_rng(40 + K)
    B, T, C = 16, 4, 512
    w = f16_round(rng.standard_normal((K, C)) / np.sqrt(K))
    b = f16_round(rng.standard_normal(C) * 0.3)
    cache_g = torch.zeros(B, K - 1, C, dtype=H, device="cuda")
    cache_o = np.zeros((B, K - 1, C))
    for _ in range(5):
        x = f16_round(rng.standard_normal((B, T, C)))
        L = rng.integers(0, T + 1, size=B).astype(np.int32)
        y = torch.empty(B, T, C, dtype=H, device="cuda")
        dw.dwconv1d_stream_fwd(dev(x, H), dev(w), dev(b), y, cache_g, dev(L))
        torch.cuda.synchronize()
        ry, cache_o = oracle.dwconv1d_stream_fwd(x, w, b, cache_o, L)
        assert_f16_close(y.float().cpu().numpy(), ry)
        assert np.array_equal(cache_g.float().cpu().numpy(), cache_o)


def run_conv2d(d, stride, pads):
    x = d["x"]
    B, T, F, C = x.shape
    KT, KF = d["w"].shape[:2]
    To, Fo = dw.conv2d_out_shape(T, F, KT, KF, stride, pads)
    L = d["lengths"]
    xg = to_dev(x)
    y = Guarded((B, To, Fo, C), H)
    ol = torch.empty(B, dtype=torch.int32, device="cuda")
    dw.dwconv2d_fwd(xg.t, dev(d["w"]), dev(d["bias"]), y.t, dev(L), ol, stride, pads)
    torch.cuda.synchronize()
    y.check_slack()
    ry, rol = oracle.dwconv2d_fwd(x, d["w"], d["bias"], L, stride, pads)
    assert_f16_close(y.numpy(), ry)
    assert np.array_equal(ol.cpu().numpy(), rol)
    gy = to_dev(d["dy"])
    dx = Guarded((B, T, F, C), H)
    dw.dwconv2d_bwd_dx(gy.t, dev(d["w"]), dx.t, dev(L), stride, pads)
    torch.cuda.synchronize()
    dx.check_slack()
    assert_f16_close(dx.numpy(), oracle.dwconv2d_bwd_dx(d["dy"], d["w"], L, T, F, stride, pads))
    gw, gb = Guarded((KT, KF, C), torch.float32), Guarded((C,), torch.float32)
    n = dw.dwconv2d_bwd_dw_workspace_size(B, T, F, C, KT, KF, stride, pads)
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    dw.dwconv2d_bwd_dw(xg.t, gy.t, gw.t, gb.t, dev(L), stride, pads, ws)
    torch.cuda.synchronize()
    grads_close((gw.numpy(), gb.numpy()), oracle.dwconv2d_bwd_dw(x, d["dy"], KT, KF, L, stride, pads))


def test_conv2d_subsampler_stage_workload():
    To, Fo = dw.conv2d_out_shape(750, 20, 3, 3, (2, 2), (1, 1, 1))
    d = conv2d_inputs(16, 750, 20, 256, 3, 3, dtype="f16", len_range=(375, 750), seed=5, dy_shape=(16, To, Fo, 256))
    run_conv2d(d, (2, 2), (1, 1, 1))


@pytest.mark.parametrize("KT,KF,stride,pads,C", [(3, 3, (1, 1), (2, 0, 1), 64), (5, 3, (2, 2), (2, 2, 1), 16),
                                                 (3, 3, (2, 1), (1, 1, 1), 6), (3, 3, (2, 2), (2, 0, 1), 40)])
def test_conv2d_general(KT, KF, stride, pads, C):
    T, F = 29, 11
    To, Fo = dw.conv2d_out_shape(T, F, KT, KF, stride, pads)
    d = conv2d_inputs(3, T, F, C, KT, KF, dtype="f16", len_range=(0, T), seed=KT * 7 + C, dy_shape=(3, To, Fo, C))
    d["lengths"][0], d["lengths"][1] = T, 0
    run_conv2d(d, stride, pads)


@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("B,T,F,C", [(16, 3000, 80, 256), (2, 37, 81, 300), (2, 23, 9, 3)])
def test_subsampler_f16_output(B, T, F, C, causal):
    d = subsample_inputs(B, T, F, C, len_range=(T // 2, T), seed=T + C)
    T4, F4 = dw.subsample_out_shape(T, F)
    out = Guarded((B, T4, F4, C), H)
    ol = torch.empty(B, dtype=torch.int32, device="cuda")
    dw.dw_subsample_fwd(dev(d["mel"]), dev(d["w0"]), dev(d["b0"]), dev(d["w1"]), dev(d["b1"]), out.t,
                        dev(d["lengths"]), ol, causal)
    torch.cuda.synchronize()
    out.check_slack()
    ref, rl = oracle.dw_subsample_fwd(d["mel"], d["w0"], d["b0"], d["w1"], d["b1"], d["lengths"], causal)
    assert_f16_close(out.numpy(), ref)
    assert np.array_equal(ol.cpu().numpy(), rl)


@pytest.mark.parametrize("B,T,F,C", [(4, 600, 80, 256), (2, 37, 81, 300)])
def test_subsampler_backward_f16_dout(B, T, F, C):
    d = subsample_inputs(B, T, F, C, len_range=(T // 2, T), seed=7 + C)
    T4, F4 = dw.subsample_out_shape(T, F)
    dout = f16_round(np.random.default_rng(C).standard_normal((B, T4, F4, C)))
    g = Guarded(dout.shape, H)
    g.t.copy_(torch.from_numpy(dout).to(H))
    outs = [Guarded((3, 3, C), torch.float32), Guarded((C,), torch.float32),
            Guarded((3, 3, C), torch.float32), Guarded((C,), torch.float32)]
    ws = torch.empty(max(dw.dw_subsample_bwd_workspace_size(B, T, F, C), 16), dtype=torch.uint8, device="cuda")
    dw.dw_subsample_bwd(dev(d["mel"]), dev(d["w0"]), dev(d["b0"]), dev(d["w1"]), g.t, dev(d["lengths"]),
                        *[o.t for o in outs], 0, ws)
    torch.cuda.synchronize()
    ref = oracle.dw_subsample_bwd(d["mel"], d["w0"], d["b0"], d["w1"], dout, d["lengths"], 0)
    # kink budget at |z| <= 2^-16 S: the rounding bound of z's float32 / TF32-split evaluation
    kdw0, kdb0 = oracle.dw_subsample_bwd_kinks(d["mel"], d["w0"], d["b0"], d["w1"], dout, d["lengths"], 0,
                                               0.0, 2.0 ** -16)
    for name, o, r, k in zip(("dw0", "db0", "dw1", "db1"), outs, ref, (kdw0, kdb0, 0.0, 0.0)):
        err = np.abs(o.numpy() - r)
        assert np.all(err <= 1e-5 * max(rms(r), 1e-6) + k), (name, float(err.max()))
