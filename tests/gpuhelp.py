"""Helpers for the GPU parity tests: device copies of the seeded inputs, guarded output
buffers (sentinel-filled slack before and after, checked after every call) and the error
measures the tolerances are stated in."""
from __future__ import annotations

import numpy as np
import torch

SENTINEL_BITS = {torch.bfloat16: 0x7FA5, torch.float32: 0x7FC0A5A5}
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
        idt = torch.int16 if dtype == torch.bfloat16 else torch.int32
        bits = SENTINEL_BITS[dtype]
        if idt == torch.int16 and bits > 0x7FFF:
            bits -= 0x10000
        self.raw = torch.full((n + 2 * SLACK + offset,), bits, dtype=idt, device="cuda")
        self.buf = self.raw.view(dtype)
        self.t = self.buf[SLACK + offset:SLACK + offset + n].view(*shape)

    def check_slack(self):
        bits = SENTINEL_BITS[self.dtype]
        idt = torch.int16 if self.dtype == torch.bfloat16 else torch.int32
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


def assert_bf16_close(got, ref, tol=2e-2):
    """bf16 I/O bar: max |gpu - oracle| <= 2e-2 absolute (float32 accumulation)."""
    e = max_abs(got, ref)
    assert e <= tol, f"max abs error {e:.3g} > {tol}"
    return e


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
