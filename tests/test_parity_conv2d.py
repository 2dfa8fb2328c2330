"""GPU parity of the general depthwise conv2d (dwconv2d_fwd, dwconv2d_bwd_dx, dwconv2d_bwd_dw)
against the fp64 CPU oracle, element by element, through the C ABI.

Workload: the subsampler's later depthwise stage, channels-last [16, 750, 20, 256] bf16 with a
3x3 stride-2 window, symmetric (1|1) and causal (2|0) time padding, frequency pad 1 ->
[16, 375, 10, 256], in full.  Edge cases: windows 1x1, 3x3, 5x3, 2x4, 3x1 and 4x4 (the runtime
path), strides 1, 2 and 3 per axis, symmetric, causal and zero pads, C that takes 4-, 2- and
1-channel vectors, T below KT (no output rows), len 0 and len T, no lengths, float32, misaligned
buffers (narrow path); out_lengths exact; dW/dbias bitwise reproducible.

Bars: outputs and dx at the bf16 or float32 I/O bar with masked rows +0.0; dW/dbias <= 2e-2
absolute and <= 1e-5 * RMS (float32 accumulation of O(1e4) products of O(1) values).
"""
import numpy as np
import pytest
import torch

import oracle
import speech_encoder_depthwise_b200 as dw
from gpuhelp import Guarded, assert_bf16_close, assert_f32_close, dev, max_abs, rms
from synth import conv2d_inputs

pytestmark = pytest.mark.gpu
TD = {"bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from speech_encoder_depthwise_b200 import build
    build.build()
    dw.lib()


def make(B, T, F, C, KT, KF, stride, pads, dtype, len_range, seed):
    To, Fo = dw.conv2d_out_shape(T, F, KT, KF, stride, pads)
    d = conv2d_inputs(B, T, F, C, KT, KF, dtype=dtype, len_range=len_range, seed=seed, dy_shape=(B, To, Fo, C))
    return d, To, Fo


def to_dev(a, dtype, offset):
    g = Guarded(a.shape, TD[dtype], offset=offset)
    g.t.copy_(torch.from_numpy(np.ascontiguousarray(a)).to(TD[dtype]))
    return g


def close(dtype, got, ref):
    (assert_f32_close if dtype == "f32" else assert_bf16_close)(got, ref)


def masked_rows_zero(got, lo):
    for b, L in enumerate(lo):
        tail = got[b, int(L):]
        assert np.all(tail == 0.0) and not np.any(np.signbit(tail)), f"item {b}: masked rows not +0.0"


def run_case(d, To, Fo, stride, pads, dtype, offset=0, check_bwd=True, with_bias=True):
    x = d["x"]
    B, T, F, C = x.shape
    KT, KF = d["w"].shape[:2]
    L = d["lengths"]
    bias = d["bias"] if with_bias else None
    # forward
    xg = to_dev(x, dtype, offset)
    y = Guarded((B, To, Fo, C), TD[dtype], offset=offset)
    ol = torch.full((B + 2,), -7, dtype=torch.int32, device="cuda")  # one guard word each side
    dw.dwconv2d_fwd(xg.t, dev(d["w"]), dev(bias), y.t, dev(L), ol[1:B + 1], stride, pads)
    torch.cuda.synchronize()
    y.check_slack()
    assert int(ol[0]) == -7 and int(ol[B + 1]) == -7, "out_lengths written out of bounds"
    ry, rol = oracle.dwconv2d_fwd(x, d["w"], bias, L, stride, pads)
    got = y.numpy()
    close(dtype, got, ry)
    assert np.array_equal(ol[1:B + 1].cpu().numpy(), rol), "out_lengths differ"
    masked_rows_zero(got, rol)
    if not check_bwd:
        return
    # data gradient
    gy = to_dev(d["dy"], dtype, offset)
    dx = Guarded((B, T, F, C), TD[dtype], offset=offset)
    dw.dwconv2d_bwd_dx(gy.t, dev(d["w"]), dx.t, dev(L), stride, pads)
    torch.cuda.synchronize()
    dx.check_slack()
    rdx = oracle.dwconv2d_bwd_dx(d["dy"], d["w"], L, T, F, stride, pads)
    gdx = dx.numpy()
    close(dtype, gdx, rdx)
    masked_rows_zero(gdx, np.full(B, T) if L is None else np.clip(L, 0, T))
    # weight and bias gradients
    gw, gb = run_dw(xg.t, gy.t, L, KT, KF, stride, pads)
    rdw, rdb = oracle.dwconv2d_bwd_dw(x, d["dy"], KT, KF, L, stride, pads)
    for g, r in ((gw, rdw), (gb, rdb)):
        e = max_abs(g, r)
        assert e <= 2e-2 and e <= 1e-5 * max(rms(r), 1e-6), (e, rms(r))


def run_dw(xt, gyt, L, KT, KF, stride, pads):
    B, T, F, C = xt.shape
    gw = Guarded((KT, KF, C), torch.float32)
    gb = Guarded((C,), torch.float32)
    n = dw.dwconv2d_bwd_dw_workspace_size(B, T, F, C, KT, KF, stride, pads)
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    dw.dwconv2d_bwd_dw(xt, gyt, gw.t, gb.t, dev(L), stride, pads, ws)
    torch.cuda.synchronize()
    gw.check_slack()
    gb.check_slack()
    return gw.numpy(), gb.numpy()


@pytest.mark.parametrize("pads", [(1, 1, 1), (2, 0, 1)], ids=["symmetric", "causal"])
def test_subsampler_stage_workload(pads):
    d, To, Fo = make(16, 750, 20, 256, 3, 3, (2, 2), pads, "bf16", (375, 750), seed=5)
    assert (To, Fo) == (375, 10)
    run_case(d, To, Fo, (2, 2), pads, "bf16")


EDGE = []
for dtype in ("bf16", "f32"):
    for (KT, KF) in ((1, 1), (3, 3), (5, 3), (2, 4), (3, 1), (4, 4)):
        for stride in ((1, 1), (2, 2), (3, 2), (2, 1)):
            for padk in ("sym", "causal", "zero"):
                EDGE.append((dtype, KT, KF, stride, padk))


def pads_of(kind, KT, KF):
    if kind == "sym":
        return ((KT - 1) // 2, KT - 1 - (KT - 1) // 2, (KF - 1) // 2)
    if kind == "causal":
        return (KT - 1, 0, (KF - 1) // 2)
    return (0, 0, 0)


@pytest.mark.parametrize("dtype,KT,KF,stride,padk", EDGE)
def test_edge_cases(dtype, KT, KF, stride, padk):
    seed = KT * 1000 + KF * 100 + stride[0] * 10 + stride[1]
    rng = np.random.default_rng(seed)
    C = int(rng.choice([8, 6, 3]))       # 4-, 2- and 1-channel vectors
    pads = pads_of(padk, KT, KF)
    d, To, Fo = make(3, 23, 9, C, KT, KF, stride, pads, dtype, (0, 23), seed)
    d["lengths"][0], d["lengths"][1] = 23, 0
    run_case(d, To, Fo, stride, pads, dtype)


@pytest.mark.parametrize("C", [1, 5, 130, 520])
def test_channel_counts(C):
    d, To, Fo = make(2, 31, 12, C, 3, 3, (2, 2), (1, 1, 1), "bf16", (5, 31), seed=C)
    run_case(d, To, Fo, (2, 2), (1, 1, 1), "bf16")


def test_no_lengths_and_no_bias():
    d, To, Fo = make(2, 17, 11, 16, 3, 3, (2, 2), (1, 1, 1), "f32", None, seed=3)
    run_case(d, To, Fo, (2, 2), (1, 1, 1), "f32", with_bias=False)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_misaligned_buffers_take_the_narrow_path(dtype):
    d, To, Fo = make(2, 20, 10, 64, 3, 3, (2, 2), (2, 0, 1), dtype, (7, 20), seed=11)
    run_case(d, To, Fo, (2, 2), (2, 0, 1), dtype, offset=1)


def test_window_longer_than_the_input():
    """T + pads < KT: no output rows; out_lengths all 0, dx all +0.0, dW and dbias zero."""
    d, To, Fo = make(2, 2, 8, 8, 5, 3, (1, 1), (1, 0, 1), "bf16", (0, 2), seed=4)
    assert To == 0
    run_case(d, To, Fo, (1, 1), (1, 0, 1), "bf16")


def test_weight_gradient_is_bitwise_reproducible():
    d, To, Fo = make(4, 200, 20, 256, 3, 3, (2, 2), (1, 1, 1), "bf16", (100, 200), seed=9)
    xt, gyt = dev(d["x"], torch.bfloat16), dev(d["dy"], torch.bfloat16)
    a = run_dw(xt, gyt, d["lengths"], 3, 3, (2, 2), (1, 1, 1))
    b = run_dw(xt, gyt, d["lengths"], 3, 3, (2, 2), (1, 1, 1))
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
