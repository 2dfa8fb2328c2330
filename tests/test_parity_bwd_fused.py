"""GPU parity of the one-pass backward (dwconv1d_bwd: the data gradient and the weight/bias
gradients from one read of dy) against the fp64 CPU oracle's two gradient functions, element by
element, through the C ABI.

Workloads: the training-size backward (32x1500x1024, K=9, bf16, symmetric) and the conformer
backward (16x1500x512, K=9, bf16), each in full; edge cases: every width with a fused instance
(1, 2, 3, 4, 5, 7, 9, 15) and widths without one (6, 20: the two-kernel path), symmetric, causal
and zero left pads, T below K and ragged tails, len 0 and T, C=520 (a partial channel tile),
float32, misaligned buffers (narrow path); results must also be bitwise reproducible.

Bars as for the separate gradients: dx at the bf16 or float32 I/O bar with masked frames +0.0;
dW/dbias <= 2e-2 absolute and <= 1e-5 * RMS.
"""
import numpy as np
import pytest
import torch

import oracle
import speech_encoder_depthwise_b200 as dw
from gpuhelp import Guarded, assert_bf16_close, assert_f32_close, assert_masked_zero, dev, max_abs, rms
from synth import conv1d_inputs, symmetric_pad_left

pytestmark = pytest.mark.gpu
TD = {"bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from speech_encoder_depthwise_b200 import build
    build.build()
    dw.lib()


def gpu_bwd(d, dtype, pad_left, K, offset=0):
    x = Guarded(d["x"].shape, TD[dtype], offset=offset)
    x.t.copy_(torch.from_numpy(np.ascontiguousarray(d["x"])).to(TD[dtype]))
    g = Guarded(d["dy"].shape, TD[dtype], offset=offset)
    g.t.copy_(torch.from_numpy(np.ascontiguousarray(d["dy"])).to(TD[dtype]))
    B, T, C = d["x"].shape
    dx = Guarded((B, T, C), TD[dtype], offset=offset)
    gw = Guarded((K, C), torch.float32)
    gb = Guarded((C,), torch.float32)
    nws = dw.dwconv1d_bwd_dw_workspace_size(B, T, C, K)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
    dw.dwconv1d_bwd(x.t, g.t, dev(d["w"]), dx.t, gw.t, gb.t, dev(d["lengths"]), pad_left, ws)
    torch.cuda.synchronize()
    for buf in (dx, gw, gb):
        buf.check_slack()
    return dx.numpy(), gw.numpy(), gb.numpy()


def check_all(d, dtype, pad_left, K, got):
    gdx, gdw, gdb = got
    T = d["x"].shape[1]
    ref = oracle.dwconv1d_bwd_dx(d["dy"], d["w"], d["lengths"], pad_left)
    (assert_f32_close if dtype == "f32" else assert_bf16_close)(gdx, ref)
    assert_masked_zero(gdx, d["lengths"], T)
    rdw, rdb = oracle.dwconv1d_bwd_dw(d["x"], d["dy"], K, d["lengths"], pad_left)
    for g, r in ((gdw, rdw), (gdb, rdb)):
        e = max_abs(g, r)
        assert e <= 2e-2 and e <= 1e-5 * max(rms(r), 1e-6), (e, rms(r))


def test_training_workload():
    d = conv1d_inputs(32, 1500, 1024, 9, dtype="bf16", len_range=(750, 1500), seed=4, with_dy=True)
    check_all(d, "bf16", 4, 9, gpu_bwd(d, "bf16", 4, 9))


def test_conformer_workload():
    d = conv1d_inputs(16, 1500, 512, 9, dtype="bf16", len_range=(750, 1500), seed=1, with_dy=True)
    check_all(d, "bf16", 4, 9, gpu_bwd(d, "bf16", 4, 9))


EDGE = []
for dtype in ("bf16", "f32"):
    for K in (1, 2, 3, 4, 5, 6, 7, 9, 15, 20):
        for (B, T, C) in ((3, 5, 8), (2, 70, 128), (2, 300, 520), (1, 1, 16)):
            EDGE.append((dtype, K, B, T, C))


@pytest.mark.parametrize("dtype,K,B,T,C", EDGE)
def test_edge_cases(dtype, K, B, T, C):
    rng = np.random.default_rng(K * 1000 + T * 10 + C)
    d = conv1d_inputs(B, T, C, K, dtype=dtype, len_range=(0, T), seed=int(rng.integers(1 << 30)), with_dy=True)
    if B >= 2:
        d["lengths"][0] = T
        d["lengths"][1] = 0 if T > 4 else d["lengths"][1]
    for pl in sorted({symmetric_pad_left(K), K - 1, 0}):
        check_all(d, dtype, pl, K, gpu_bwd(d, dtype, pl, K))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_misaligned_buffers_take_the_narrow_path(dtype):
    d = conv1d_inputs(2, 50, 64, 9, dtype=dtype, len_range=(20, 50), seed=7, with_dy=True)
    check_all(d, dtype, 4, 9, gpu_bwd(d, dtype, 4, 9, offset=1))


def test_results_are_bitwise_reproducible():
    d = conv1d_inputs(8, 700, 512, 9, dtype="bf16", len_range=(300, 700), seed=12, with_dy=True)
    a = gpu_bwd(d, "bf16", 4, 9)
    b = gpu_bwd(d, "bf16", 4, 9)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
