"""Helpers for the GPU parity tests: device copies of the seeded inputs, guarded output
buffers (sentinel-filled slack before and after, checked after every call) and the error
measures the tolerances are stated in."""
from __future__ import annotations

import numpy as np
import torch

SENTINEL_BITS = {torch.bfloat16: 0x7FA5, torch.float16: 0x7DA5, torch.float32: 0x7FC0A5A5}
SLACK = 64  # elements of guard band on each side (keeps 16-byte alignment)


def dev(a, dtype=torch.float32):
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(device="cuda", dtype=dtype if t.dtype != torch.int32 else torch.int32)


class Guarded:
    """An output tensor inside a larger buffer whose slack holds a sentinel bit pattern."""

    def __init__(self, shape, dtype, offset=0):
        n = int(np.prod(shape))
        self.dtype = dtype
        self.n = n
        self.offset = offset
        idt = torch.int32 if dtype == torch.float32 else torch.int16
        bits = SENTINEL_BITS[dtype]
        if idt == torch.int16 and bits > 0x7FFF:
            bits -= 0x10000
        self.raw = torch.full((n + 2 * SLACK + offset,), bits, dtype=idt, device="cuda")
        self.buf = self.raw.view(dtype)
        self.t = self.buf[SLACK + offset:SLACK + offset + n].view(*shape)

    def check_slack(self):
        bits = SENTINEL_BITS[self.dtype]
        idt = torch.int32 if self.dtype == torch.float32 else torch.int16
        if idt == torch.int16 and bits > 0x7FFF:
            bits -= 0x10000
        head = self.raw[:SLACK + self.offset]
        tail = self.raw[SLACK + self.offset + self.n:]
        assert bool((head == bits).all()), "write before the output buffer"
        assert bool((tail == bits).all()), "write after the output buffer"

    def numpy(self):
        return self.t.float().cpu().numpy().astype(np.float64)


def max_abs(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def rms(a):
    a = np.asarray(a, np.float64)
    return float(np.sqrt(np.mean(a * a))) if a.size else 0.0


def bf16_ulp(v):
    """Spacing of bf16 numbers at |v| (8 significant bits): 2^(e-8) for |v| in [2^(e-1), 2^e)."""
    v = np.abs(np.asarray(v, np.float64))
    _, e = np.frexp(np.maximum(v, 2.0 ** -126))
    return np.ldexp(1.0, e - 8)


def assert_bf16_close(got, ref, tol=2e-2):
    """bf16 I/O bar, element by element: |gpu - oracle| <= max(2e-2, one bf16 ulp of the oracle value).

    2e-2 absolute is the stated bar for bf16 I/O with float32 accumulation.  Where |y| >= 4 the
    spacing of bf16 numbers (0.031 in [4, 8), 0.0625 in [8, 16)) exceeds it, and no bf16 value
    lies within 2e-2 of every exact result; there the bar is one unit of the output precision.
    On top of that bar, the result must be faithfully rounded: within one bf16 ulp of the exact
    value everywhere (plus 1e-5 for the float32 accumulation error of O(1) terms, which matters
    only where cancellation makes the result tiny), which is what float32 accumulation and one
    round-to-nearest-even store give.
    """
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if got.size == 0:
        return 0.0
    err = np.abs(got - ref)
    ulp = bf16_ulp(ref)
    bar = np.maximum(tol, ulp)
    bad = err > bar
    if bad.any():
        i = np.unravel_index(np.argmax(err - bar), err.shape)
        raise AssertionError(f"{int(bad.sum())} elements beyond the bf16 bar; worst at {i}: "
                             f"gpu {got[i]!r} oracle {ref[i]!r} err {err[i]:.3g} bar {bar[i]:.3g}")
    unfaithful = err >= ulp + 1e-5
    assert not unfaithful.any(), f"{int(unfaithful.sum())} elements not faithfully rounded to bf16"
    return float(err.max())


def f16_ulp(v):
    """Spacing of IEEE float16 numbers at |v| (11 significant bits; subnormal spacing 2^-24)."""
    v = np.abs(np.asarray(v, np.float64))
    _, e = np.frexp(np.maximum(v, 2.0 ** -14))
    return np.ldexp(1.0, e - 11)


def assert_f16_close(got, ref):
    """fp16 I/O bar (no figure is stated for fp16; this one follows from the arithmetic): float32
    accumulation and one round-to-nearest-even store give a faithfully rounded result, so
    |gpu - oracle| < ulp_f16(oracle) + 1e-5 element by element (the 1e-5 covers the float32
    accumulation error of O(1) terms where cancellation makes the result tiny)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if got.size == 0:
        return 0.0
    err = np.abs(got - ref)
    bar = f16_ulp(ref) + 1e-5
    bad = err >= bar
    if bad.any():
        i = np.unravel_index(np.argmax(err - bar), err.shape)
        raise AssertionError(f"{int(bad.sum())} elements beyond the fp16 bar; worst at {i}: "
                             f"gpu {got[i]!r} oracle {ref[i]!r} err {err[i]:.3g} bar {bar[i]:.3g}")
    return float(err.max())


def assert_close(dtype, got, ref):
    """The I/O bar of `dtype` ("f32", "bf16" or "f16")."""
    if dtype == "f32":
        return assert_f32_close(got, ref)
    if dtype == "f16":
        return assert_f16_close(got, ref)
    return assert_bf16_close(got, ref)


def assert_f32_close(got, ref, rel=1e-5):
    """float32 I/O bar: max |gpu - oracle| <= 1e-5 * RMS(oracle)."""
    e = max_abs(got, ref)
    bound = rel * max(rms(ref), 1e-30)
    assert e <= bound, f"max abs error {e:.3g} > {bound:.3g} (= {rel} * RMS)"
    return e


def assert_masked_zero(got, lengths, T):
    """Frames at or beyond len_b are +0.0 exactly."""
    if lengths is None:
        return
    for b, L in enumerate(lengths):
        L = min(max(int(L), 0), T)
        tail = got[b, L:]
        assert np.all(tail == 0.0) and not np.any(np.signbit(tail)), f"item {b}: masked frames not +0.0"
