"""GPU parity on batches with more items than the balanced work deals take, through the C ABI.

The conv1d weight gradient and the one-pass backward deal equal spans of the valid frames from
per-item tables for up to 1024 items; larger batches take the unit-dealt pipelined kernels (and
their cluster reduction).  The fused subsampler balances its units with per-item prefix tables
for up to 4096 items and deals them round robin beyond (and then does not warm L2 with the
lengths).  The subsampler backward lists each block's units for any batch.  These tests run
each of those paths on short items (lengths from 0 to T, so empty and partly masked items
occur) and compare element by element with the fp64 oracle.

Bars as the other parity tests: bf16 / fp16 outputs faithfully rounded (max(2e-2, one ulp)),
float32 within 1e-5 * RMS, masked frames +0.0, weight gradients within 2e-2 and 1e-5 * RMS (the
subsampler backward's dw0 / db0 plus the oracle's kink budget).
"""
import numpy as np
import pytest
import torch

import oracle
import speech_encoder_depthwise_b200 as dw
from gpuhelp import Guarded, assert_close, assert_masked_zero, dev, max_abs, rms
from synth import bf16_round, conv1d_inputs, subsample_inputs, symmetric_pad_left

pytestmark = pytest.mark.gpu
TD = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from speech_encoder_depthwise_b200 import build
    build.build()
    dw.lib()


def assert_dw_close(got, ref):
    e = max_abs(got, ref)
    assert e <= 2e-2 and e <= 1e-5 * max(rms(ref), 1e-6), f"weight gradient error {e:.3g} (RMS {rms(ref):.3g})"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,K", [(1100, 9), (1030, 4)])
def test_conv1d_more_than_1024_items(B, K, dtype):
    T, C = 40, 64
    pl = symmetric_pad_left(K)
    d = conv1d_inputs(B, T, C, K, dtype=dtype, len_range=(0, T), seed=B + K, with_dy=True)
    L = d["lengths"]
    x, g = dev(d["x"], TD[dtype]), dev(d["dy"], TD[dtype])
    w, bias, ln = dev(d["w"]), dev(d["bias"]), dev(L)
    y, dx = Guarded(x.shape, TD[dtype]), Guarded(x.shape, TD[dtype])
    gw, gb = Guarded((K, C), torch.float32), Guarded((C,), torch.float32)
    ws = torch.empty(max(dw.dwconv1d_bwd_dw_workspace_size(B, T, C, K), 16), dtype=torch.uint8, device="cuda")
    dw.dwconv1d_fwd(x, w, bias, y.t, ln, pl)
    dw.dwconv1d_bwd_dx(g, w, dx.t, ln, pl)
    dw.dwconv1d_bwd_dw(x, g, gw.t, gb.t, ln, pl, ws)
    torch.cuda.synchronize()
    for o in (y, dx, gw, gb):
        o.check_slack()
    assert dw.dw_device_error() == 0
    assert_close(dtype, y.numpy(), oracle.dwconv1d_fwd(d["x"], d["w"], d["bias"], L, pl))
    assert_masked_zero(y.numpy(), L, T)
    rdx = oracle.dwconv1d_bwd_dx(d["dy"], d["w"], L, pl)
    assert_close(dtype, dx.numpy(), rdx)
    assert_masked_zero(dx.numpy(), L, T)
    rw, rb = oracle.dwconv1d_bwd_dw(d["x"], d["dy"], K, L, pl)
    assert_dw_close(gw.numpy(), rw)
    assert_dw_close(gb.numpy(), rb)
    # the one-pass backward on the same batch: dx and the weight gradients from one read of dy
    dx1 = Guarded(x.shape, TD[dtype])
    gw1, gb1 = Guarded((K, C), torch.float32), Guarded((C,), torch.float32)
    dw.dwconv1d_bwd(x, g, w, dx1.t, gw1.t, gb1.t, ln, pl, ws)
    torch.cuda.synchronize()
    for o in (dx1, gw1, gb1):
        o.check_slack()
    assert_close(dtype, dx1.numpy(), rdx)
    assert_masked_zero(dx1.numpy(), L, T)
    assert_dw_close(gw1.numpy(), rw)
    assert_dw_close(gb1.numpy(), rb)


@pytest.mark.parametrize("simt", [False, True])
@pytest.mark.parametrize("causal", [False, True])
def test_subsampler_more_than_4096_items(causal, simt):
    B, T, F, C = 4200, 12, 16, 128
    d = subsample_inputs(B, T, F, C, len_range=(0, T), seed=90 + causal)
    T4, F4 = dw.subsample_out_shape(T, F)
    out = Guarded((B, T4, F4, C), torch.bfloat16)
    ol = torch.full((B,), -5, dtype=torch.int32, device="cuda")
    fn = dw.dw_subsample_fwd_simt if simt else dw.dw_subsample_fwd
    fn(dev(d["mel"]), dev(d["w0"]), dev(d["b0"]), dev(d["w1"]), dev(d["b1"]), out.t, dev(d["lengths"]), ol, causal)
    torch.cuda.synchronize()
    out.check_slack()
    assert dw.dw_device_error() == 0
    ref, rl = oracle.dw_subsample_fwd(d["mel"], d["w0"], d["b0"], d["w1"], d["b1"], d["lengths"], causal)
    assert np.array_equal(ol.cpu().numpy(), rl)
    got = out.numpy()
    assert_close("bf16", got, ref)
    for b, L4 in enumerate(rl):
        tail = got[b, L4:]
        assert np.all(tail == 0.0) and not np.any(np.signbit(tail))


def test_subsampler_backward_many_items():
    B, T, F, C = 1500, 12, 16, 64
    d = subsample_inputs(B, T, F, C, len_range=(0, T), seed=95)
    T4, F4 = dw.subsample_out_shape(T, F)
    dout = bf16_round(np.random.default_rng(96).standard_normal((B, T4, F4, C)).astype(np.float32))
    g = dev(dout, torch.bfloat16)
    grads = [Guarded(s, torch.float32) for s in ((3, 3, C), (C,), (3, 3, C), (C,))]
    ws = torch.empty(max(dw.dw_subsample_bwd_workspace_size(B, T, F, C), 16), dtype=torch.uint8, device="cuda")
    dw.dw_subsample_bwd(dev(d["mel"]), dev(d["w0"]), dev(d["b0"]), dev(d["w1"]), g, dev(d["lengths"]),
                        *[o.t for o in grads], False, ws)
    torch.cuda.synchronize()
    for o in grads:
        o.check_slack()
    assert dw.dw_device_error() == 0
    ref = oracle.dw_subsample_bwd(d["mel"], d["w0"], d["b0"], d["w1"], dout, d["lengths"], False)
    kdw0, kdb0 = oracle.dw_subsample_bwd_kinks(d["mel"], d["w0"], d["b0"], d["w1"], dout, d["lengths"], False,
                                               0.0, 2.0 ** -16)
    for name, o, r, k in zip(("dw0", "db0", "dw1", "db1"), grads, ref, (kdw0, kdb0, 0.0, 0.0)):
        err = np.abs(o.numpy() - r)
        bound = 1e-5 * max(rms(r), 1e-6) + k
        assert np.all(err <= bound), f"{name}: max error {err.max():.3g}"
