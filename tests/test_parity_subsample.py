"""GPU parity of the fused depthwise-striding subsampler front against the fp64 CPU oracle,
element by element, through the C ABI.

Full size: mel [16, 3000, 80] -> out [16, 750, 20, 256] bf16, lengths uniform in
[1500, 3000], symmetric and causal (time pad 2|0): the configuration the benchmark times.
Small cases: T and F from 1 up (odd and even), C not a multiple of 64 (1, 3, 100, 300),
C up to 512 (several channel tiles), F up to 200 (several 20-column blocks),
float32 output, len 0 and len T, unaligned output (narrow store path), guard bands.

Both entry points are checked at full size: dw_subsample_fwd (conv0 on the tensor cores where
the output rows are 16-byte aligned) and dw_subsample_fwd_simt (every step on the FP32 pipes);
the small cases also run dw_subsample_fwd_simt on shapes the tensor-core kernel would take.

Bars: bf16 output max|err| <= 2e-2 absolute; float32 output max|err| <= 1e-5 * RMS(oracle);
masked rows exactly +0.0; out_lengths bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
import speech_encoder_depthwise_b200 as dw
from gpuhelp import Guarded, assert_bf16_close, assert_f32_close, dev
from synth import subsample_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from speech_encoder_depthwise_b200 import build
    build.build()
    dw.lib()


def gpu_subsample(d, causal, out_dtype=torch.bfloat16, offset=0, with_lengths=True, simt=False):
    mel = dev(d["mel"])
    B, T, F = mel.shape
    C = d["w0"].shape[-1]
    T4, F4 = dw.subsample_out_shape(T, F)
    out = Guarded((B, T4, F4, C), out_dtype, offset=offset)
    ol = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    fn = dw.dw_subsample_fwd_simt if simt else dw.dw_subsample_fwd
    fn(mel, dev(d["w0"]), dev(d["b0"]), dev(d["w1"]), dev(d["b1"]), out.t,
       dev(d["lengths"]) if with_lengths else None, ol, causal)
    torch.cuda.synchronize()
    out.check_slack()
    return out.numpy(), ol.cpu().numpy()


def check_masked_rows(got, out_lengths):
    for b, L4 in enumerate(out_lengths):
        tail = got[b, L4:]
        assert np.all(tail == 0.0) and not np.any(np.signbit(tail))


@pytest.mark.parametrize("simt", [False, True])
@pytest.mark.parametrize("causal", [False, True])
def test_subsampler_full_workload(causal, simt):
    """Both entry points: dw_subsample_fwd (tensor-core conv0) and dw_subsample_fwd_simt (all FP32)."""
    d = subsample_inputs(16, 3000, 80, 256, len_range=(1500, 3000), seed=3)
    ref, rl = oracle.dw_subsample_fwd(d["mel"], d["w0"], d["b0"], d["w1"], d["b1"], d["lengths"], causal)
    got, gl = gpu_subsample(d, causal, simt=simt)
    assert got.shape == ref.shape == (16, 750, 20, 256)
    assert_bf16_close(got, ref)
    np.testing.assert_array_equal(gl, rl)
    check_masked_rows(got, gl)


SMALL = [(1, 1, 1, 1), (2, 2, 3, 3), (2, 5, 7, 64), (3, 9, 80, 100), (2, 64, 80, 256), (2, 37, 81, 300),
         (1, 130, 16, 128), (2, 33, 9, 1), (1, 4, 4, 2),
         # tensor-core path: several column blocks, an odd number of channel tiles, two channel
         # groups, a single output column
         (2, 45, 200, 384), (1, 70, 80, 512), (2, 23, 3, 32)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,T,F,C", SMALL)
@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
def test_subsampler_small_cases(B, T, F, C, causal, out_dtype):
    d = subsample_inputs(B, T, F, C, len_range=(0, T), seed=T * 100 + F + C)
    d["lengths"][0] = T
    if B > 2:
        d["lengths"][1] = 0
    ref, rl = oracle.dw_subsample_fwd(d["mel"], d["w0"], d["b0"], d["w1"], d["b1"], d["lengths"], causal)
    td = torch.float32 if out_dtype == "f32" else torch.bfloat16
    got, gl = gpu_subsample(d, causal, out_dtype=td)
    if out_dtype == "f32":
        assert_f32_close(got, ref)
    else:
        assert_bf16_close(got, ref)
    np.testing.assert_array_equal(gl, rl)
    check_masked_rows(got, gl)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,T,F,C", [(2, 45, 200, 384), (1, 70, 80, 512), (2, 23, 3, 32), (2, 64, 80, 256)])
def test_subsampler_simt_entry_on_aligned_shapes(B, T, F, C, causal):
    d = subsample_inputs(B, T, F, C, len_range=(0, T), seed=T * 100 + F + C)
    d["lengths"][0] = T
    ref, rl = oracle.dw_subsample_fwd(d["mel"], d["w0"], d["b0"], d["w1"], d["b1"], d["lengths"], causal)
    for td, close in ((torch.float32, assert_f32_close), (torch.bfloat16, assert_bf16_close)):
        got, gl = gpu_subsample(d, causal, out_dtype=td, simt=True)
        close(got, ref)
        np.testing.assert_array_equal(gl, rl)
        check_masked_rows(got, gl)


def test_subsampler_unaligned_output_and_no_lengths():
    d = subsample_inputs(2, 50, 20, 64, len_range=(50, 50), seed=5)
    ref, rl = oracle.dw_subsample_fwd(d["mel"], d["w0"], d["b0"], d["w1"], d["b1"], None, False)
    got, gl = gpu_subsample(d, False, offset=1, with_lengths=False)
    assert_bf16_close(got, ref)
    np.testing.assert_array_equal(gl, rl)


def test_subsampler_mel_beyond_len_is_ignored():
    """The kernel counts mel frames at or beyond len_b as zero itself."""
    d = subsample_inputs(2, 40, 16, 64, len_range=(10, 30), seed=6)
    a, _ = gpu_subsample(d, False)
    d2 = dict(d)
    m = d["mel"].copy()
    for b in range(2):
        m[b, d["lengths"][b]:] = 5.0
    d2["mel"] = m
    b_, _ = gpu_subsample(d2, False)
    np.testing.assert_array_equal(a, b_)


def test_subsampler_causal_ignores_future():
    d = subsample_inputs(1, 120, 16, 64, len_range=(120, 120), seed=7)
    base, _ = gpu_subsample(d, True)
    d2 = dict(d)
    m = d["mel"].copy()
    m[:, 4 * 10 + 1:] = -2.0   # out row i reads mel rows <= 4 i
    d2["mel"] = m
    got, _ = gpu_subsample(d2, True)
    np.testing.assert_array_equal(got[:, :11], base[:, :11])
