"""Seeded synthetic inputs for the depthwise-conv hot path.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark.  It only draws numbers: it holds none of the convolution arithmetic.

Recipe (one ``numpy.random.default_rng(seed)`` per workload):

* conv1d: draw ``x`` ~ N(0, 1), then ``w[K, C]`` ~ N(0, 1/K), then ``bias[C]``
  ~ N(0, 0.1), then ``lengths[B]`` uniform on the inclusive integer range, then
  (backward workloads only) ``dy`` ~ N(0, 1).  N(m, v) names the variance ``v``.
* subsampler: draw ``mel[B, T, F]`` ~ N(0, 1), then ``w0[3, 3, C]`` ~ N(0, 1/9),
  ``b0`` ~ N(0, 0.1), ``w1[3, 3, C]`` ~ N(0, 1/9), ``b1`` ~ N(0, 0.1), then
  ``lengths``.  Mel frames at ``t >= lengths[b]`` are then set to zero, so a
  reading that masks the mel before conv0 and one that does not agree.
* conv2d: draw ``x[B, T, F, C]`` ~ N(0, 1), then ``w[KT, KF, C]`` ~ N(0, 1/(KT KF)),
  ``bias[C]`` ~ N(0, 0.1), then ``lengths``, then (when the caller gives the output
  shape) ``dy`` ~ N(0, 1) of that shape.
* bf16 (fp16) workloads round every drawn value (data and weights) to the nearest
  bf16- (fp16-) representable float32, ties to even, so the stored 16-bit tensor and
  the float32 weights hold exactly the values the oracle reads.

All arrays are float32 (values) or int32 (lengths), C-contiguous, channels last.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_round",
    "f16_round",
    "dyadic_round",
    "bf16_bits",
    "conv1d_inputs",
    "subsample_inputs",
    "conv2d_inputs",
    "symmetric_pad_left",
    "WORKLOADS",
]


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16-representable float32 (ties to even)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).reshape(a.shape)


def f16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest IEEE float16 value (ties to even), as float32."""
    return np.ascontiguousarray(a, dtype=np.float32).astype(np.float16).astype(np.float32)


def _round_to(dtype, out, keys):
    if dtype == "bf16":
        for k in keys:
            if k in out:
                out[k] = bf16_round(out[k])
    elif dtype == "f16":
        for k in keys:
            if k in out:
                out[k] = f16_round(out[k])
    elif dtype != "f32":
        raise ValueError(f"unknown dtype {dtype!r}")


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """The upper 16 bits of bf16-representable float32 values, as uint16 (the stored bf16)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def symmetric_pad_left(K: int) -> int:
    """Left pad of the symmetric ('same') mode: floor((K-1)/2); the extra pad of an even K goes right."""
    return (K - 1) // 2


def _normal(rng, shape, var):
    return (rng.standard_normal(shape, dtype=np.float32) * np.float32(np.sqrt(var))).astype(np.float32)


def conv1d_inputs(B, T, C, K, *, dtype="bf16", len_range=None, seed=0, with_dy=False):
    """Inputs of one depthwise conv1d workload.

    Returns a dict with ``x[B,T,C]``, ``w[K,C]``, ``bias[C]`` (float32, rounded to
    bf16 values when ``dtype == 'bf16'``), ``lengths[B]`` (int32, or None when
    ``len_range`` is None: no masking) and, with ``with_dy``, ``dy[B,T,C]``.
    """
    rng = np.random.default_rng(seed)
    x = _normal(rng, (B, T, C), 1.0)
    w = _normal(rng, (K, C), 1.0 / K)
    bias = _normal(rng, (C,), 0.1)
    lengths = None
    if len_range is not None:
        lo, hi = len_range
        lengths = rng.integers(lo, hi + 1, size=B).astype(np.int32)
    out = {"x": x, "w": w, "bias": bias, "lengths": lengths}
    if with_dy:
        out["dy"] = _normal(rng, (B, T, C), 1.0)
    _round_to(dtype, out, ("x", "w", "bias", "dy"))
    return out


def dyadic_round(a: np.ndarray, frac_bits: int) -> np.ndarray:
    """Round float32 values to the nearest multiple of 2**-frac_bits (ties to even), as float32."""
    s = np.float32(2.0 ** frac_bits)
    return (np.rint(np.asarray(a, np.float32) * s) / s).astype(np.float32)


def subsample_inputs(B, T, F, C, *, len_range, seed=3, zero_beyond_len=True, dyadic=False):
    """Inputs of one fused-subsampler workload: ``mel[B,T,F]``, ``w0,w1[3,3,C]``, ``b0,b1[C]``, ``lengths[B]``.

    ``dyadic=True`` rounds the same draws onto coarse binary grids: mel to multiples of 2**-6,
    w0 to 2**-8 and b0 to 2**-14.  Every mel value and w0 weight then has at most 11
    significant bits and every product and partial sum of conv0 is a multiple of 2**-14 below
    2**7 in magnitude, so conv0's output is exactly representable in float32 however its terms
    are split, ordered or rounded.
    """
    rng = np.random.default_rng(seed)
    mel = _normal(rng, (B, T, F), 1.0)
    w0 = _normal(rng, (3, 3, C), 1.0 / 9.0)
    b0 = _normal(rng, (C,), 0.1)
    if dyadic:
        mel = dyadic_round(np.clip(mel, -7.0, 7.0), 6)
        w0 = dyadic_round(np.clip(w0, -1.9, 1.9), 8)
        b0 = dyadic_round(b0, 14)
    w1 = _normal(rng, (3, 3, C), 1.0 / 9.0)
    b1 = _normal(rng, (C,), 0.1)
    lo, hi = len_range
    lengths = rng.integers(lo, hi + 1, size=B).astype(np.int32)
    if zero_beyond_len:
        for b in range(B):
            mel[b, max(0, int(lengths[b])):, :] = 0.0
    return {"mel": mel, "w0": w0, "b0": b0, "w1": w1, "b1": b1, "lengths": lengths}


def conv2d_inputs(B, T, F, C, KT, KF, *, dtype="bf16", len_range=None, seed=0, dy_shape=None):
    """Inputs of one depthwise conv2d workload: ``x[B,T,F,C]``, ``w[KT,KF,C]``, ``bias[C]``,
    ``lengths[B]`` (None without ``len_range``) and, given ``dy_shape``, ``dy``."""
    rng = np.random.default_rng(seed)
    out = {"x": _normal(rng, (B, T, F, C), 1.0), "w": _normal(rng, (KT, KF, C), 1.0 / (KT * KF)),
           "bias": _normal(rng, (C,), 0.1), "lengths": None}
    if len_range is not None:
        lo, hi = len_range
        out["lengths"] = rng.integers(lo, hi + 1, size=B).astype(np.int32)
    if dy_shape is not None:
        out["dy"] = _normal(rng, tuple(dy_shape), 1.0)
    _round_to(dtype, out, ("x", "w", "bias", "dy"))
    return out


# The five workloads, shaped like the ones the pages run (the parakeet conformer
# conv at K=9, a kernel-width sweep, NeMo's depthwise-striding subsampler and a
# training-size backward).  Seed = workload index.
WORKLOADS = {
    "fwd_f32_small": dict(kind="conv1d", B=1, T=200, C=256, K=9, dtype="f32", len_range=None,
                          pad="symmetric", seed=0),
    "fwd_bf16_B16_T1500_C512_K9": dict(kind="conv1d", B=16, T=1500, C=512, K=9, dtype="bf16",
                                       len_range=(750, 1500), pad="symmetric", seed=1),
    "fwd_bf16_causal_sweep": dict(kind="conv1d", B=32, T=750, C=1024, Ks=(3, 4, 5, 9, 15),
                                  dtype="bf16", len_range=(375, 750), pad="causal", seed=2,
                                  odd_case=dict(C=520, K=7)),
    "subsample_B16_T3000_F80_C256": dict(kind="subsample", B=16, T=3000, F=80, C=256,
                                         len_range=(1500, 3000), seed=3),
    "bwd_bf16_B32_T1500_C1024_K9": dict(kind="conv1d_bwd", B=32, T=1500, C=1024, K=9,
                                        dtype="bf16", len_range=(750, 1500), pad="symmetric",
                                        seed=4),
}
