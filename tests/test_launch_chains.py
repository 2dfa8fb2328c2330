"""GPU tests of kernels launched back to back, each reading what the call before it wrote.

Every pipelined kernel starts under programmatic dependent launch: it may begin while the
previous kernel in the stream drains, warms L2 with what it reads first, and waits
(griddepcontrol.wait) before its first real read.  A read placed before that wait would see
stale data only when the producer is the immediately preceding kernel, which the one-call
parity tests never arrange.  Here each stage is queued right after the one that produces its
input (no host synchronisation in between) into buffers that held different values before, and
each stage is checked against the fp64 oracle evaluated on the GPU's own input to that stage:

- conv1d forward -> forward -> data gradient and weight gradient (outputs as inputs);
- the fused subsampler writing out_lengths into a buffer holding wrong lengths, then conv1d and
  conv2d over its output with those lengths (lengths as inputs);
- the subsampler's output as the dout of its own backward.

Bars are the parity tests': bf16 outputs faithfully rounded (max(2e-2, one bf16 ulp)), masked
frames +0.0, weight gradients within 2e-2 and 1e-5 * RMS.
"""
import numpy as np
import pytest
import torch

import oracle
import speech_encoder_depthwise_b200 as dw
from gpuhelp import assert_bf16_close, assert_masked_zero, dev, max_abs, rms
from synth import conv1d_inputs, conv2d_inputs, subsample_inputs, symmetric_pad_left

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from speech_encoder_depthwise_b200 import build
    build.build()
    dw.lib()


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def assert_dw_close(got, ref):
    e = max_abs(got, ref)
    assert e <= 2e-2 and e <= 1e-5 * max(rms(ref), 1e-30), f"weight gradient error {e:.3g} (RMS {rms(ref):.3g})"


@pytest.mark.parametrize("rep", range(3))
def test_conv1d_chain_outputs_as_inputs(rep):
    """Conformer shape: y1 = fwd(x), y2 = fwd(y1), dx = bwd_dx(y2), (gw, gb) = bwd_dw(x, y2), queued
    back to back into buffers pre-filled with a large constant."""
    B, T, C, K = 16, 1500, 512, 9
    pl = symmetric_pad_left(K)
    d = conv1d_inputs(B, T, C, K, dtype="bf16", len_range=(T // 2, T), seed=40 + rep)
    x = dev(d["x"], torch.bfloat16)
    w, bias, ln = dev(d["w"]), dev(d["bias"]), dev(d["lengths"])
    fill = lambda: torch.full((B, T, C), 1000.0, dtype=torch.bfloat16, device="cuda")
    y1, y2, dx = fill(), fill(), fill()
    gw = torch.full((K, C), 1000.0, device="cuda")
    gb = torch.full((C,), 1000.0, device="cuda")
    ws = torch.empty(max(dw.dwconv1d_bwd_dw_workspace_size(B, T, C, K), 16), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    dw.dwconv1d_fwd(x, w, bias, y1, ln, pl)
    dw.dwconv1d_fwd(y1, w, bias, y2, ln, pl)
    dw.dwconv1d_bwd_dx(y2, w, dx, ln, pl)
    dw.dwconv1d_bwd_dw(x, y2, gw, gb, ln, pl, ws)
    torch.cuda.synchronize()
    assert dw.dw_device_error() == 0
    L = d["lengths"]
    g1, g2 = f64(y1), f64(y2)
    assert_bf16_close(g1, oracle.dwconv1d_fwd(d["x"], d["w"], d["bias"], L, pl))
    assert_bf16_close(g2, oracle.dwconv1d_fwd(g1, d["w"], d["bias"], L, pl))
    assert_bf16_close(f64(dx), oracle.dwconv1d_bwd_dx(g2, d["w"], L, pl))
    for got in (g1, g2, f64(dx)):
        assert_masked_zero(got, L, T)
    rw, rb = oracle.dwconv1d_bwd_dw(d["x"], g2, K, L, pl)
    assert_dw_close(gw.cpu().numpy(), rw)
    assert_dw_close(gb.cpu().numpy(), rb)


@pytest.mark.parametrize("causal", [False, True])
def test_lengths_written_by_the_previous_kernel(causal):
    """The subsampler writes out_lengths over wrong values (every frame valid); conv1d forward, its
    weight gradient and conv2d forward then take those lengths, and the subsampler's output, at once."""
    B, T, F, C = 16, 3000, 80, 256
    d = subsample_inputs(B, T, F, C, len_range=(T // 2, T), seed=50 + causal)
    T4, F4 = dw.subsample_out_shape(T, F)
    out = torch.full((B, T4, F4, C), 1000.0, dtype=torch.bfloat16, device="cuda")
    ol = torch.full((B,), T4, dtype=torch.int32, device="cuda")  # wrong until the subsampler writes it
    K, Cc = 9, F4 * C
    pl = symmetric_pad_left(K)
    rng = np.random.default_rng(60 + causal)
    w1d = (rng.standard_normal((K, Cc)) / 3.0).astype(np.float32)
    b1d = (rng.standard_normal(Cc) * 0.1).astype(np.float32)
    c2 = conv2d_inputs(B, T4, F4, C, 3, 3, dtype="bf16", seed=70 + causal)
    stride, pads = (2, 2), (1, 1, 1)
    To, Fo = dw.conv2d_out_shape(T4, F4, 3, 3, stride, pads)
    y1 = torch.full((B, T4, Cc), 1000.0, dtype=torch.bfloat16, device="cuda")
    y2 = torch.full((B, To, Fo, C), 1000.0, dtype=torch.bfloat16, device="cuda")
    ol2 = torch.full((B,), -3, dtype=torch.int32, device="cuda")
    gw = torch.full((K, Cc), 1000.0, device="cuda")
    gb = torch.full((Cc,), 1000.0, device="cuda")
    ws = torch.empty(max(dw.dwconv1d_bwd_dw_workspace_size(B, T4, Cc, K), 16), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    dw.dw_subsample_fwd(dev(d["mel"]), dev(d["w0"]), dev(d["b0"]), dev(d["w1"]), dev(d["b1"]), out,
                        dev(d["lengths"]), ol, causal)
    x1 = out.view(B, T4, Cc)
    dw.dwconv1d_fwd(x1, dev(w1d), dev(b1d), y1, ol, pl)
    dw.dwconv1d_bwd_dw(x1, y1, gw, gb, ol, pl, ws)
    dw.dwconv2d_fwd(out, dev(c2["w"]), dev(c2["bias"]), y2, ol, ol2, stride, pads)
    torch.cuda.synchronize()
    assert dw.dw_device_error() == 0

    ref_out, ref_ol = oracle.dw_subsample_fwd(d["mel"], d["w0"], d["b0"], d["w1"], d["b1"], d["lengths"], causal)
    assert np.array_equal(ol.cpu().numpy(), ref_ol)
    g_out = f64(out)
    assert_bf16_close(g_out, ref_out)
    L4 = ref_ol
    g1 = f64(y1)
    assert_bf16_close(g1, oracle.dwconv1d_fwd(g_out.reshape(B, T4, Cc), w1d, b1d, L4, pl))
    assert_masked_zero(g1, L4, T4)  # frames past the true lengths: the stale lengths would fill them
    rw, rb = oracle.dwconv1d_bwd_dw(g_out.reshape(B, T4, Cc), g1, K, L4, pl)
    assert_dw_close(gw.cpu().numpy(), rw)
    assert_dw_close(gb.cpu().numpy(), rb)
    ref2, ref_ol2 = oracle.dwconv2d_fwd(g_out, c2["w"], c2["bias"], L4, stride, pads)
    assert np.array_equal(ol2.cpu().numpy(), ref_ol2)
    assert_bf16_close(f64(y2), ref2)


def test_subsampler_output_as_backward_dout():
    """The subsampler's bf16 output, still in flight, is the dout of its own backward (the
    tensor-core backward reads it with tensor copies); the weight gradients are checked against
    the oracle on the GPU's output, with the oracle's kink budget as in the backward parity tests."""
    B, T, F, C = 4, 400, 80, 256
    d = subsample_inputs(B, T, F, C, len_range=(T // 2, T), seed=80)
    T4, F4 = dw.subsample_out_shape(T, F)
    out = torch.full((B, T4, F4, C), 1000.0, dtype=torch.bfloat16, device="cuda")
    ol = torch.empty(B, dtype=torch.int32, device="cuda")
    grads = [torch.full(s, 1000.0, device="cuda") for s in ((3, 3, C), (C,), (3, 3, C), (C,))]
    ws = torch.empty(max(dw.dw_subsample_bwd_workspace_size(B, T, F, C), 16), dtype=torch.uint8, device="cuda")
    mel, w0, b0, w1, b1, ln = (dev(d[k]) for k in ("mel", "w0", "b0", "w1", "b1", "lengths"))
    torch.cuda.synchronize()
    dw.dw_subsample_fwd(mel, w0, b0, w1, b1, out, ln, ol, False)
    dw.dw_subsample_bwd(mel, w0, b0, w1, out, ln, *grads, False, ws)
    torch.cuda.synchronize()
    assert dw.dw_device_error() == 0
    dout = f64(out)
    ref = oracle.dw_subsample_bwd(d["mel"], d["w0"], d["b0"], d["w1"], dout, d["lengths"], False)
    kdw0, kdb0 = oracle.dw_subsample_bwd_kinks(d["mel"], d["w0"], d["b0"], d["w1"], dout, d["lengths"], False,
                                               0.0, 2.0 ** -16)
    for name, g, r, k in zip(("dw0", "db0", "dw1", "db1"), grads, ref, (kdw0, kdb0, 0.0, 0.0)):
        err = np.abs(g.cpu().numpy().astype(np.float64) - r)
        bound = 1e-5 * max(rms(r), 1e-6) + k
        assert np.all(err <= bound), f"{name}: max error {err.max():.3g}"
