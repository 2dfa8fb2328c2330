"""GPU parity at wide channel counts, through the C ABI.

The conv1d kernels tile C in 128-channel slabs, and each block keeps one slab for all of its
work; the fused subsampler deals channel tiles to blocks in groups of two.  These cases run
many slabs, a ragged last slab, a row width that is not a multiple of 16 bytes (narrow path),
and subsampler channel counts that give three and four channel groups (the last group half
empty), each against the fp64 oracle element by element.  Bars as the other parity tests.
"""
import numpy as np
import pytest
import torch

import oracle
import speech_encoder_depthwise_b200 as dw
from gpuhelp import Guarded, assert_close, assert_masked_zero, dev, max_abs, rms
from synth import bf16_round, conv1d_inputs, subsample_inputs, symmetric_pad_left

pytestmark = pytest.mark.gpu
TD = {"bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from speech_encoder_depthwise_b200 import build
    build.build()
    dw.lib()


def assert_dw_close(got, ref):
    e = max_abs(got, ref)
    assert e <= 2e-2 and e <= 1e-5 * max(rms(ref), 1e-6), f"weight gradient error {e:.3g} (RMS {rms(ref):.3g})"


@pytest.mark.parametrize("C,dtype,K", [(8192, "bf16", 9), (4104, "bf16", 15), (2050, "f32", 9), (1032, "f32", 4)])
def test_conv1d_wide(C, dtype, K):
    B, T = 3, 60
    pl = symmetric_pad_left(K)
    d = conv1d_inputs(B, T, C, K, dtype=dtype, len_range=(T // 3, T), seed=C + K, with_dy=True)
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
    assert_close(dtype, dx.numpy(), oracle.dwconv1d_bwd_dx(d["dy"], d["w"], L, pl))
    rw, rb = oracle.dwconv1d_bwd_dw(d["x"], d["dy"], K, L, pl)
    assert_dw_close(gw.numpy(), rw)
    assert_dw_close(gb.numpy(), rb)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("C", [640, 1024, 136])
def test_subsampler_channel_groups(C, causal):
    B, T, F = 2, 64, 80
    d = subsample_inputs(B, T, F, C, len_range=(T // 2, T), seed=C + causal)
    d["lengths"][0] = T
    T4, F4 = dw.subsample_out_shape(T, F)
    out = Guarded((B, T4, F4, C), torch.bfloat16)
    ol = torch.full((B,), -5, dtype=torch.int32, device="cuda")
    dw.dw_subsample_fwd(dev(d["mel"]), dev(d["w0"]), dev(d["b0"]), dev(d["w1"]), dev(d["b1"]), out.t,
                        dev(d["lengths"]), ol, causal)
    torch.cuda.synchronize()
    out.check_slack()
    assert dw.dw_device_error() == 0
    ref, rl = oracle.dw_subsample_fwd(d["mel"], d["w0"], d["b0"], d["w1"], d["b1"], d["lengths"], causal)
    assert np.array_equal(ol.cpu().numpy(), rl)
    assert_close("bf16", out.numpy(), ref)


@pytest.mark.parametrize("C", [640, 1024])
def test_subsampler_backward_channel_groups(C):
    B, T, F = 2, 48, 80
    d = subsample_inputs(B, T, F, C, len_range=(T // 2, T), seed=C + 7)
    T4, F4 = dw.subsample_out_shape(T, F)
    dout = bf16_round(np.random.default_rng(C).standard_normal((B, T4, F4, C)).astype(np.float32))
    grads = [Guarded(s, torch.float32) for s in ((3, 3, C), (C,), (3, 3, C), (C,))]
    ws = torch.empty(max(dw.dw_subsample_bwd_workspace_size(B, T, F, C), 16), dtype=torch.uint8, device="cuda")
    dw.dw_subsample_bwd(dev(d["mel"]), dev(d["w0"]), dev(d["b0"]), dev(d["w1"]), dev(dout, torch.bfloat16),
                        dev(d["lengths"]), *[o.t for o in grads], False, ws)
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
