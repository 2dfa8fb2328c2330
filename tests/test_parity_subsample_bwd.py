"""GPU parity of the subsampler backward (dw_subsample_bwd: the gradients of sum(out * dout) with
respect to w0, b0, w1, b1) against the fp64 CPU oracle, through the C ABI.

Bars: dw1 and db1 within 1e-5 * RMS(oracle) (float32 accumulation).  dw0 and db0 within
1e-5 * RMS(oracle) plus the oracle's kink budget.  The ReLU derivative [z > 0] is decided on a
recomputed float32 z, so at h pixels where |z| is within the rounding error of that evaluation the
GPU and the float64 oracle may decide differently; each such pixel can move dw0[p,q,c] by at most
|dz| |mel tap| and db0[c] by |dz|, and the budget is that sum per element.

The rounding bound: z = b0 + sum_t mel_t w0_t is evaluated either by float32 FMAs (error below
10 * 2^-24 * S, S = |b0| + sum_t |mel_t w0_t|) or on the tensor cores from TF32 words, each operand
split into a high word and its remainder: per product the dropped lo*lo term and the truncation of
the remainders stay below 3 * 2^-20 of the product, and the float32 accumulation of the 29 split
terms adds at most 29 * 2^-22 * S.  Together that is below 41 * 2^-22 * S < 1e-5 * S; the tests use
|z| <= 2^-16 * S (KINK_REL), a margin of 1.5.

At the benchmark's full size the tests draw the inputs on dyadic grids (synth's ``dyadic``): every
product and partial sum of z is then exactly representable in float32 and in the TF32 split, the
GPU's z equals the exact z, both sides take the same ReLU decisions, and the kink budget is
exactly 0: dw0 / db0 are held to 1e-5 * RMS alone, so a dropped or doubled h pixel fails.

Workloads: the benchmark's subsampler shape (mel 16x3000x80, C=256, lengths in [1500, 3000]) with
bf16 dout, symmetric and causal; small cases with T and F from 1, odd C, C past one channel
group, float32 dout, misaligned dout, len 0, no lengths; bitwise reproducibility.
"""
import numpy as np
import pytest
import torch

import oracle
import speech_encoder_depthwise_b200 as dw
from gpuhelp import Guarded, dev, max_abs, rms
from synth import bf16_round, f16_round, subsample_inputs

pytestmark = pytest.mark.gpu
KINK_REL = 2.0 ** -16


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from speech_encoder_depthwise_b200 import build
    build.build()
    dw.lib()


def gpu_bwd(d, dout, causal, dtype=torch.bfloat16, offset=0, with_lengths=True):
    B, T, F = d["mel"].shape
    C = d["w0"].shape[-1]
    g = Guarded(dout.shape, dtype, offset=offset)
    g.t.copy_(torch.from_numpy(np.ascontiguousarray(dout)).to(dtype))
    outs = [Guarded((3, 3, C), torch.float32), Guarded((C,), torch.float32),
            Guarded((3, 3, C), torch.float32), Guarded((C,), torch.float32)]
    n = dw.dw_subsample_bwd_workspace_size(B, T, F, C)
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    dw.dw_subsample_bwd(dev(d["mel"]), dev(d["w0"]), dev(d["b0"]), dev(d["w1"]), g.t,
                        dev(d["lengths"]) if with_lengths else None, *[o.t for o in outs], causal, ws)
    torch.cuda.synchronize()
    for o in outs + [g]:
        o.check_slack()
    return [o.numpy() for o in outs]


def check(d, dout, causal, got, with_lengths=True, exact_z=False):
    """exact_z: the inputs are on the dyadic grids, so both sides decide [z > 0] alike (no budget)."""
    L = d["lengths"] if with_lengths else None
    ref = oracle.dw_subsample_bwd(d["mel"], d["w0"], d["b0"], d["w1"], dout, L, causal)
    if exact_z:
        kdw0, kdb0 = 0.0, 0.0
    else:
        kdw0, kdb0 = oracle.dw_subsample_bwd_kinks(d["mel"], d["w0"], d["b0"], d["w1"], dout, L, causal,
                                                   0.0, KINK_REL)
    ratios = []
    for name, g, r, k in zip(("dw0", "db0", "dw1", "db1"), got, ref, (kdw0, kdb0, 0.0, 0.0)):
        bar = 1e-5 * max(rms(r), 1e-6)
        bound = bar + k
        err = np.abs(g - r)
        assert np.all(err <= bound), f"{name}: max error {err.max():.3g}, bound {np.min(bound):.3g}..."
        ratios.append(float(np.max(k)) / bar)
    return ratios


def rounded_dout(d, causal, seed, dtype="bf16"):
    B, T, F = d["mel"].shape
    C = d["w0"].shape[-1]
    T4, F4 = oracle.subsample_out_shape(T, F, causal)
    g = np.random.default_rng(seed).standard_normal((B, T4, F4, C)).astype(np.float32)
    return {"bf16": bf16_round, "f16": f16_round}.get(dtype, lambda x: x)(g)


def assert_z_exact(d, items=1, rows=64):
    """The dyadic inputs' claim on a sample: z summed in float32, in two orders, equals float64."""
    mel, w0, b0 = d["mel"][:items, :rows], d["w0"].reshape(9, -1), d["b0"]
    B, T, F = mel.shape
    mp = np.pad(mel, ((0, 0), (1, 1), (1, 1)))
    taps = [mp[:, p:p + T:2, q:q + F:2] for p in range(3) for q in range(3)]
    z64 = b0.astype(np.float64) + sum(t[..., None].astype(np.float64) * w0[i] for i, t in enumerate(taps))
    fw = np.float32(0) + b0
    for i, t in enumerate(taps):
        fw = (fw + t[..., None] * w0[i]).astype(np.float32)
    bw = np.zeros_like(fw)
    for i, t in reversed(list(enumerate(taps))):
        bw = (bw + t[..., None] * w0[i]).astype(np.float32)
    bw = (bw + b0).astype(np.float32)
    assert np.array_equal(fw.astype(np.float64), z64) and np.array_equal(bw.astype(np.float64), z64)


@pytest.mark.parametrize("causal", [False, True])
def test_full_workload(causal):
    """Full size on dyadic inputs: no kink budget, dw0 / db0 within 1e-5 * RMS."""
    d = subsample_inputs(16, 3000, 80, 256, len_range=(1500, 3000), seed=3, dyadic=True)
    assert_z_exact(d)
    dout = rounded_dout(d, causal, 30 + causal)
    ratios = check(d, dout, causal, gpu_bwd(d, dout, causal), exact_z=True)
    print(f"kink budget / bar at full size (dw0, db0): {ratios[0]:.3g}, {ratios[1]:.3g}")


def test_full_workload_continuous_inputs():
    """Full size on the workload's own (continuous) draws, which also run the TF32 split's
    remainder products of conv0: dw0 / db0 carry the kink budget here."""
    d = subsample_inputs(16, 3000, 80, 256, len_range=(1500, 3000), seed=3)
    dout = rounded_dout(d, False, 30)
    ratios = check(d, dout, False, gpu_bwd(d, dout, False))
    print(f"kink budget / bar at full size, continuous inputs (dw0, db0): {ratios[0]:.3g}, {ratios[1]:.3g}")


SMALL = [(1, 1, 1, 1), (2, 5, 7, 3), (3, 9, 80, 100), (2, 37, 81, 300), (1, 130, 16, 128), (2, 33, 9, 1),
         (2, 64, 80, 257)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,T,F,C", SMALL)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_small_cases(B, T, F, C, causal, dtype):
    d = subsample_inputs(B, T, F, C, len_range=(0, T), seed=T * 100 + F + C)
    d["lengths"][0] = T
    if B > 2:
        d["lengths"][1] = 0
    dout = rounded_dout(d, causal, T + C, dtype)
    got = gpu_bwd(d, dout, causal, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32)
    check(d, dout, causal, got)


def test_misaligned_dout_and_no_lengths():
    d = subsample_inputs(2, 50, 20, 64, len_range=(50, 50), seed=5)
    dout = rounded_dout(d, False, 6)
    check(d, dout, False, gpu_bwd(d, dout, False, offset=1, with_lengths=False), with_lengths=False)


def test_results_are_bitwise_reproducible():
    d = subsample_inputs(4, 400, 80, 256, len_range=(200, 400), seed=8)
    dout = rounded_dout(d, False, 9)
    a = gpu_bwd(d, dout, False)
    b = gpu_bwd(d, dout, False)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


# Shapes the tensor-core kernel takes (16-bit dout, C a multiple of 8): one channel tile and a
# ragged second one, F2 past one 40-column block, T from 1, many short items, odd unit counts.
TC = [(1, 1, 1, 8), (2, 37, 81, 136), (3, 130, 100, 256), (5, 61, 80, 64), (7, 9, 3, 16), (1, 400, 80, 384),
      (1, 9, 1270, 8), (1, 9, 1290, 8)]  # 16 column blocks (the most a unit entry holds), then 17 (SIMT)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,T,F,C", TC)
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_tensor_core_shapes(B, T, F, C, causal, dtype):
    d = subsample_inputs(B, T, F, C, len_range=(0, T), seed=T * 7 + F + C)
    d["lengths"][0] = T
    dout = rounded_dout(d, causal, T + F + C, dtype)
    got = gpu_bwd(d, dout, causal, dtype=torch.bfloat16 if dtype == "bf16" else torch.float16)
    check(d, dout, causal, got)


def test_tensor_core_full_workload_f16_causal():
    d = subsample_inputs(16, 3000, 80, 256, len_range=(1500, 3000), seed=13, dyadic=True)
    dout = rounded_dout(d, True, 14, "f16")
    check(d, dout, True, gpu_bwd(d, dout, True, dtype=torch.float16), exact_z=True)
