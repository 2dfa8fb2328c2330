"""GPU parity of the packed-batch conv1d (dwconv1d_fwd_packed, dwconv1d_bwd_dx_packed,
dwconv1d_bwd_dw_packed) against
the fp64 CPU oracle, element by element, through the C ABI.

Workload: the conformer batch (16 sequences, lengths U[750, 1500], C=512, K=9, symmetric)
packed back to back, in bf16, fp16 and float32.  Edge cases: empty sequences and sequences
shorter than the window, causal K=15, runtime K=6, C that takes 2- and 1-channel vectors,
misaligned buffers (general kernel), more sequences than one launch's table holds (1500 short
ones), and rows after offsets[B] (must stay untouched).  Bars as the padded kernels: bf16
|err| <= max(2e-2, 1 ulp) and faithful, fp16 faithful, float32 <= 1e-5 * RMS; dW/dbias <= 2e-2
absolute and <= 1e-5 * RMS, bitwise reproducible.
"""
import numpy as np
import pytest
import torch

import oracle
import speech_encoder_depthwise_b200 as dw
from gpuhelp import Guarded, assert_close, dev, max_abs, rms
from synth import conv1d_inputs, symmetric_pad_left

pytestmark = pytest.mark.gpu
TD = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from speech_encoder_depthwise_b200 import build
    build.build()
    dw.lib()


def packed_case(lens, C, K, dtype, seed, extra_rows=0):
    """Sequences of the given lengths drawn like the padded workloads, packed into [N, C]."""
    lens = np.asarray(lens, np.int32)
    d = conv1d_inputs(len(lens), int(max(lens.max(), 1)), C, K, dtype=dtype, len_range=None, seed=seed,
                      with_dy=True)
    x = np.concatenate([d["x"][b, :lens[b]] for b in range(len(lens))] + [d["x"][0, :extra_rows]])
    dy = np.concatenate([d["dy"][b, :lens[b]] for b in range(len(lens))] + [d["dy"][0, :extra_rows]])
    offsets = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return x, dy, d["w"], d["bias"], offsets


def run(x, dy, w, bias, offsets, pl, dtype, offset=0):
    N, C = x.shape
    covered = int(offsets[-1])
    xg = Guarded((N, C), TD[dtype], offset=offset)
    xg.t.copy_(torch.from_numpy(x).to(TD[dtype]))
    y = Guarded((N, C), TD[dtype], offset=offset)
    y.t.fill_(7.0)
    dw.dwconv1d_fwd_packed(xg.t, dev(w), dev(bias), y.t, dev(offsets), pl)
    torch.cuda.synchronize()
    y.check_slack()
    got = y.numpy()
    assert_close(dtype, got[:covered], oracle.dwconv1d_fwd_packed(x, w, bias, offsets, pl)[:covered])
    assert np.all(got[covered:] == 7.0), "rows after the last sequence were written"
    gy = Guarded((N, C), TD[dtype], offset=offset)
    gy.t.copy_(torch.from_numpy(dy).to(TD[dtype]))
    dx = Guarded((N, C), TD[dtype], offset=offset)
    dx.t.fill_(7.0)
    dw.dwconv1d_bwd_dx_packed(gy.t, dev(w), dx.t, dev(offsets), pl)
    torch.cuda.synchronize()
    dx.check_slack()
    gdx = dx.numpy()
    assert_close(dtype, gdx[:covered], oracle.dwconv1d_bwd_dx_packed(dy, w, offsets, pl)[:covered])
    assert np.all(gdx[covered:] == 7.0)
    K = w.shape[0]
    gw, gb = gpu_dw_packed(xg.t, gy.t, offsets, K, pl)
    rw, rb = oracle.dwconv1d_bwd_dw_packed(x[:covered], dy[:covered], K, offsets, pl)
    for g, r in ((gw, rw), (gb, rb)):
        e = max_abs(g, r)
        assert e <= 2e-2 and e <= 1e-5 * max(rms(r), 1e-6), (e, rms(r))


def gpu_dw_packed(xt, gyt, offsets, K, pl):
    N, C = xt.shape
    gw, gb = Guarded((K, C), torch.float32), Guarded((C,), torch.float32)
    n = dw.dwconv1d_bwd_dw_packed_workspace_size(len(offsets) - 1, N, C, K)
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    dw.dwconv1d_bwd_dw_packed(xt, gyt, gw.t, gb.t, dev(offsets), pl, ws)
    torch.cuda.synchronize()
    gw.check_slack()
    gb.check_slack()
    return gw.numpy(), gb.numpy()


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
def test_conformer_batch_packed(dtype):
    rng = np.random.default_rng(1)
    lens = rng.integers(750, 1501, size=16)
    run(*packed_case(lens, 512, 9, dtype, seed=1), 4, dtype)


@pytest.mark.parametrize("K,pl", [(15, 14), (6, 2), (9, 8), (1, 0)])
def test_widths_and_short_sequences(K, pl):
    lens = [40, 0, 3, 1, 0, 77, K - 1 if K > 1 else 1, 130]
    run(*packed_case(lens, 256, K, "bf16", seed=K), pl, "bf16")


@pytest.mark.parametrize("C", [130, 7])
def test_narrow_channel_vectors(C):
    run(*packed_case([50, 9, 0, 33], C, 9, "bf16", seed=C), 4, "bf16")


def test_misaligned_buffers_take_the_general_kernel():
    run(*packed_case([60, 5, 41], 64, 9, "f16", seed=5), 4, "f16", offset=1)


def test_more_sequences_than_one_table():
    rng = np.random.default_rng(3)
    lens = rng.integers(0, 12, size=1500)
    run(*packed_case(lens, 64, 9, "bf16", seed=3), 4, "bf16")


def test_rows_after_the_last_sequence_are_untouched():
    run(*packed_case([20, 31], 128, 9, "bf16", seed=9, extra_rows=17), 4, "bf16")


def test_packed_equals_padded_gpu_on_valid_frames():
    """The packed kernel and the padded kernel on the same sequences agree bit for bit."""
    rng = np.random.default_rng(11)
    B, T, C, K = 8, 400, 512, 9
    lens = rng.integers(100, T + 1, size=B).astype(np.int32)
    d = conv1d_inputs(B, T, C, K, dtype="bf16", len_range=None, seed=11)
    yp = torch.empty(B, T, C, dtype=torch.bfloat16, device="cuda")
    dw.dwconv1d_fwd(dev(d["x"], torch.bfloat16), dev(d["w"]), dev(d["bias"]), yp, dev(lens), 4)
    x = np.concatenate([d["x"][b, :lens[b]] for b in range(B)])
    offsets = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    y = torch.empty(x.shape[0], C, dtype=torch.bfloat16, device="cuda")
    dw.dwconv1d_fwd_packed(dev(x, torch.bfloat16), dev(d["w"]), dev(d["bias"]), y, dev(offsets), 4)
    torch.cuda.synchronize()
    for b in range(B):
        assert torch.equal(y[offsets[b]:offsets[b + 1]], yp[b, :lens[b]])


def test_packed_weight_gradient_is_reproducible():
    rng = np.random.default_rng(21)
    x, dy, w, bias, offsets = packed_case(rng.integers(100, 900, size=12), 512, 9, "bf16", seed=21)
    xt, gt = dev(x, torch.bfloat16), dev(dy, torch.bfloat16)
    a = gpu_dw_packed(xt, gt, offsets, 9, 4)
    b = gpu_dw_packed(xt, gt, offsets, 9, 4)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
