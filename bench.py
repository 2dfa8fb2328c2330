"""Benchmark of the depthwise-convolution hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
  * depthwise conv1d forward, data gradient and weight/bias gradients on the conformer
    workload x[16, 1500, 512] bf16, K = 9, symmetric padding 4|4, lengths uniform in [750, 1500];
  * the fused depthwise-striding subsampler on mel[16, 3000, 80] fp32 -> out[16, 750, 20, 256]
    bf16, symmetric padding, lengths uniform in [1500, 3000].
Inputs are resident in device memory; three rotating input sets (about 237 MB each, larger
than L2 together and alone) keep every step's reads cold in L2.  Every kernel launch is
bracketed by CUDA events on its stream.  The value is algorithmic bytes per step (valid input
frames read, all output frames written, parameters) divided by the step time.

`--impl reference` times the CPU oracle (the only reference this path has) on a bounded
sample of the same workload.  Multi-GPU: one process per GPU (torchrun), each rank its own
batch, no collective on the data path (weak scaling); time = max over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("dwconv1d HBM GB/s & frames/s (B16 T1500 C512 K9 bf16); subsampler ms and % roofline")
CONV = dict(B=16, T=1500, C=512, K=9, pad_left=4, len_range=(750, 1500), seed=1)
SUB = dict(B=16, T=3000, F=80, C=256, causal=0, len_range=(1500, 3000), seed=3)
N_SETS = 3
WORKLOAD = ("conformer depthwise conv1d B16 T1500 C512 K9 bf16 sym 4|4, len U[750,1500]: fwd + dX + "
            "dW/dbias; fused depthwise-striding subsampler B16 T3000 F80 -> B16 T750 F20 C256 bf16 sym, "
            "len U[1500,3000]")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--e2e-steps", type=int, default=20)
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--next-rows", default="all",
                   help="comma list of the measurements after the step: the other workloads (sweep: causal "
                        "kernel-width sweep; sub: subsampler symmetric/causal, tensor-core and FP32 kernels; bwd: "
                        "training-size dX, dW and one-pass backward) and the NEXT rows (stream, conv2d, "
                        "f16_packed, sub_bwd, batch); 'all' or 'none'")
    return p.parse_args()


# ------------------------------------------------------------------ algorithmic work
def conv_work(lengths, T, C, K, esize=2):
    """Bytes and flops of the three conv1d legs (valid input frames read, all outputs written)."""
    B = len(lengths)
    valid = int(np.clip(lengths, 0, T).sum())
    params = K * C * 4 + C * 4 + B * 4
    fwd_b = valid * C * esize + B * T * C * esize + params
    dx_b = valid * C * esize + B * T * C * esize + K * C * 4 + B * 4
    dw_b = 2 * valid * C * esize + (K + 1) * C * 4 + B * 4
    fl = 2 * K * valid * C
    return dict(fwd=(fwd_b, fl), dx=(dx_b, fl), dw=(dw_b, fl + valid * C)), valid


def sub_work(lengths, T, F, C, esize=2):
    s2 = lambda n: (n - 1) // 2 + 1 if n >= 1 else 0
    T2, F2 = s2(T), s2(F)
    T4, F4 = s2(T2), s2(F2)
    B = len(lengths)
    L = np.clip(lengths, 0, T).astype(np.int64)
    L2 = np.minimum((L + 1) // 2, T2)
    L4 = np.minimum((L2 + 1) // 2, T4)
    by = int(L.sum()) * F * 4 + B * T4 * F4 * C * esize + 2 * (9 * C * 4 + C * 4) + B * 8
    fl = int(L2.sum()) * F2 * C * 18 + int(L4.sum()) * F4 * C * 18
    return by, fl, T4, F4


# ------------------------------------------------------------------ multi-rank aggregation
def max_over_ranks(value, world, device="cpu"):
    """The largest value over all ranks (the job's time is its slowest rank's)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(step_bytes_per_rank, ms_per_step, world):
    """Whole-job GB/s: every rank processes its own batch (weak scaling) in the slowest rank's time."""
    return world * step_bytes_per_rank / (ms_per_step * 1e-3) / 1e9


# ------------------------------------------------------------------ errors against the parity bars
def bf16_err_over_bar(got, ref):
    """max over elements of |gpu - oracle| / bar with the bf16 I/O bar the parity tests apply element
    by element: bar = max(2e-2, one bf16 ulp of the oracle value) (where |y| >= 4 the bf16 spacing
    exceeds 2e-2, so the bar there is one unit of the output precision).  <= 1 passes."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    _, e = np.frexp(np.maximum(np.abs(ref), 2.0 ** -126))
    bar = np.maximum(2e-2, np.ldexp(1.0, e - 8))
    return float(np.max(np.abs(got - ref) / bar)) if ref.size else 0.0


def dw_err_over_bar(got, ref):
    """|gpu - oracle| / bar for float32 weight gradients from bf16 inputs: the tests hold the max error
    to both 2e-2 absolute and 1e-5 * RMS(oracle), so bar = the smaller of the two.  <= 1 passes."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    bar = min(2e-2, 1e-5 * float(np.sqrt(np.mean(ref * ref))))
    return float(np.max(np.abs(got - ref)) / max(bar, 1e-30))


# ------------------------------------------------------------------ clocks (NVML, read only)
class ClockSampler:
    """Samples SM clock and throttle reasons in a background thread (reads only)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index):
        self.samples, self.reasons, self.ok = [], set(), False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        med = float(np.median(self.samples)) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------------ helpers
STREAM = dict(B=64, C=512, K=9, chunks=(1, 16), seed=21)


def measure_stream(dw, dev, hbm):
    """Streaming causal conv with a cache (a NEXT row, outside the step): 64 streams, C=512,
    K=9, bf16, chunks of 1 and 16 frames; 8 chunks captured in a graph, replayed.  Reports µs
    per chunk, GB/s (chunk in, output, cache in and out), frames/s and the max error of one chunk
    against the oracle."""
    import torch
    import oracle
    from synth import bf16_round
    B, C, K = STREAM["B"], STREAM["C"], STREAM["K"]
    rng = np.random.default_rng(STREAM["seed"])
    w = bf16_round(rng.standard_normal((K, C)) / np.sqrt(K))
    b = bf16_round(rng.standard_normal(C) * np.sqrt(0.1))
    gw = torch.from_numpy(w).to(dev)
    gb = torch.from_numpy(b).to(dev)
    res = {}
    for T in STREAM["chunks"]:
        xs = [bf16_round(rng.standard_normal((B, T, C))) for _ in range(8)]
        gx = [torch.from_numpy(x).to(dev, torch.bfloat16) for x in xs]
        gy = [torch.empty_like(x) for x in gx]
        cache = torch.zeros(B, K - 1, C, dtype=torch.bfloat16, device=dev)
        s = torch.cuda.Stream(dev)
        with torch.cuda.stream(s):
            dw.dwconv1d_stream_fwd(gx[0], gw, gb, gy[0], cache, None)
            torch.cuda.synchronize(dev)
            y0 = gy[0].float().cpu().numpy()
            ry, _ = oracle.dwconv1d_stream_fwd(xs[0], w, b, np.zeros((B, K - 1, C)), None)
            err = float(np.max(np.abs(y0 - ry)))
            g = torch.cuda.CUDAGraph()
            g.capture_begin()
            for i in range(8):
                dw.dwconv1d_stream_fwd(gx[i], gw, gb, gy[i], cache, None)
            g.capture_end()
            for _ in range(5):
                g.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            for _ in range(50):
                g.replay()
            e1.record(s)
        torch.cuda.synchronize(dev)
        us = e0.elapsed_time(e1) / 400 * 1e3
        by = (2 * B * T * C + 2 * B * (K - 1) * C) * 2
        res[f"chunk{T}"] = {"us": us, "GB_per_s": by / us / 1e3, "hbm_frac_of_measured": by / us / 1e3 / hbm,
                            "frames_per_s": B * T / (us * 1e-6), "alg_bytes": by, "max_abs_err": err}
        del g
    return {"workload": f"streaming causal dwconv1d with a [K-1,C] cache: {B} streams, C={C}, K={K}, bf16, "
                        "chunks of 1 and 16 frames (8 chunks per CUDA graph)", **res}


BWD = dict(B=32, T=1500, C=1024, K=9, pad_left=4, len_range=(750, 1500), seed=4)


def measure_bwd(dw, dev, hbm):
    """The training-size backward workload, 32x1500x1024 bf16, K=9, sym 4|4, len U[750,1500]:
    the data gradient (dwconv1d_bwd_dx) and the weight/bias gradients (dwconv1d_bwd_dw) as rows of
    their own, and the one-pass dwconv1d_bwd (a NEXT row), each over 3 rotating input sets
    captured in a CUDA graph.  Algorithmic bytes: dX = dy at valid frames + dx in full; dW = x and
    dy at valid frames; one pass = x and dy at valid frames + dx in full."""
    import torch
    import oracle
    from synth import conv1d_inputs
    B, T, C, K, pl = BWD["B"], BWD["T"], BWD["C"], BWD["K"], BWD["pad_left"]
    d = conv1d_inputs(B, T, C, K, dtype="bf16", len_range=BWD["len_range"], seed=BWD["seed"], with_dy=True)
    x0 = torch.from_numpy(d["x"]).to(dev, torch.bfloat16)
    g0 = torch.from_numpy(d["dy"]).to(dev, torch.bfloat16)
    xs, gs = [x0] + [x0.clone() for _ in range(2)], [g0] + [g0.clone() for _ in range(2)]
    dxs = [torch.empty_like(x0) for _ in range(3)]
    w = torch.from_numpy(d["w"]).to(dev)
    ln = torch.from_numpy(d["lengths"]).to(dev)
    gw, gb = torch.empty(K, C, device=dev), torch.empty(C, device=dev)
    ws = torch.empty(dw.dwconv1d_bwd_dw_workspace_size(B, T, C, K), dtype=torch.uint8, device=dev)
    valid = int(np.clip(d["lengths"], 0, T).sum()) * C
    by_dx = (valid + B * T * C) * 2 + K * C * 4 + B * 4
    by_dw = 2 * valid * 2 + (K + 1) * C * 4 + B * 4
    by_one = (2 * valid + B * T * C) * 2
    fl = 2 * K * valid
    t_dx = graph_us(dev, [lambda i=i: dw.dwconv1d_bwd_dx(gs[i], w, dxs[i], ln, pl) for i in range(3)])
    t_dw = graph_us(dev, [lambda i=i: dw.dwconv1d_bwd_dw(xs[i], gs[i], gw, gb, ln, pl, ws) for i in range(3)])
    t_one = graph_us(dev, [lambda i=i: dw.dwconv1d_bwd(xs[i], gs[i], w, dxs[i], gw, gb, ln, pl, ws)
                           for i in range(3)])
    # errors against the oracle: dX on items 0-1, dW/dbias over the whole batch
    dw.dwconv1d_bwd_dx(gs[0], w, dxs[0], ln, pl)
    dw.dwconv1d_bwd_dw(xs[0], gs[0], gw, gb, ln, pl, ws)
    torch.cuda.synchronize(dev)
    rdx = oracle.dwconv1d_bwd_dx(d["dy"][:2], d["w"], d["lengths"][:2], pl)
    gdx = dxs[0][:2].float().cpu().numpy()
    rdw, rdb = oracle.dwconv1d_bwd_dw(d["x"], d["dy"], K, d["lengths"], pl)
    gdw, gdb = gw.cpu().numpy(), gb.cpu().numpy()

    def row(us, by, flops):
        return {"us": us, "GB_per_s": by / us / 1e3, "frames_per_s": B * T / (us * 1e-6),
                "hbm_frac_of_measured": by / us / 1e3 / hbm, "hbm_frac_of_8TBps": by / us / 1e3 / 8000.0,
                "alg_bytes": by, "alg_flops": flops}
    rdx_row = row(t_dx, by_dx, fl)
    rdx_row.update(max_abs_err=float(np.max(np.abs(gdx - rdx))), err_over_bar=bf16_err_over_bar(gdx, rdx))
    rdw_row = row(t_dw, by_dw, fl + valid)
    rdw_row.update(max_abs_err=max(float(np.max(np.abs(gdw - rdw))), float(np.max(np.abs(gdb - rdb)))),
                   err_over_bar=max(dw_err_over_bar(gdw, rdw), dw_err_over_bar(gdb, rdb)))
    one = row(t_one, by_one, 2 * fl + valid)
    one["dx_plus_dw_as_two_launches_us"] = t_dx + t_dw
    return {"workload": f"conv1d backward {B}x{T}x{C} bf16, K={K}, sym 4|4, len U[750,1500] "
                        "(3 rotating input sets in a CUDA graph)",
            "dwconv1d_bwd_dx": rdx_row, "dwconv1d_bwd_dw": rdw_row, "dwconv1d_bwd_one_pass": one}


def measure_sub_bwd(dw, dev, hbm, fp32_tflops):
    """Subsampler backward (a NEXT row, outside the step) on the benchmark's subsampler shape,
    mel 16x3000x80, C=256, bf16 dout, symmetric: µs, and the roofline of its algorithmic work:
    mel at valid frames + dout read, 18 flop per valid h element (conv0 recomputed, dw0) and
    18 per valid output element (dh, dw1)."""
    import torch
    from synth import subsample_inputs
    B, T, F, C = SUB["B"], SUB["T"], SUB["F"], SUB["C"]
    ss = subsample_inputs(B, T, F, C, len_range=SUB["len_range"], seed=SUB["seed"])
    t = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    mel, w0, b0, w1, ln = t(ss["mel"]), t(ss["w0"]), t(ss["b0"]), t(ss["w1"]), t(ss["lengths"], torch.int32)
    T4, F4 = dw.subsample_out_shape(T, F)
    gen = torch.Generator(device=dev).manual_seed(31)
    douts = [torch.randn(B, T4, F4, C, device=dev, generator=gen).to(torch.bfloat16) for _ in range(3)]
    g = [torch.empty(3, 3, C, device=dev), torch.empty(C, device=dev), torch.empty(3, 3, C, device=dev),
         torch.empty(C, device=dev)]
    ws = torch.empty(dw.dw_subsample_bwd_workspace_size(B, T, F, C), dtype=torch.uint8, device=dev)
    s = torch.cuda.Stream(dev)
    with torch.cuda.stream(s):
        for i in range(3):
            dw.dw_subsample_bwd(mel, w0, b0, w1, douts[i], ln, *g, SUB["causal"], ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for i in range(20):
            dw.dw_subsample_bwd(mel, w0, b0, w1, douts[i % 3], ln, *g, SUB["causal"], ws)
        e1.record(s)
    torch.cuda.synchronize(dev)
    us = e0.elapsed_time(e1) / 20 * 1e3
    L = np.clip(ss["lengths"], 0, T)
    L2 = (L + 1) // 2
    L4 = (L2 + 1) // 2
    F2 = (F + 1) // 2
    by = int(L.sum()) * F * 4 + B * T4 * F4 * C * 2
    fl = int(L2.sum()) * F2 * C * 36 + int(L4.sum()) * F4 * C * 36
    t_roof = max(by / (hbm * 1e9), fl / (fp32_tflops * 1e12))
    return {"workload": "subsampler backward, mel 16x3000x80 -> C256, bf16 dout, sym, len U[1500,3000]",
            "kernel": "dw_subsample_bwd_tc_kernel (tcgen05: conv0 recompute and dw0/db0) + finalize",
            "us": us, "TFLOP_per_s": fl / (us * 1e-6) / 1e12, "roofline_frac": t_roof / (us * 1e-6),
            "alg_bytes": by, "alg_flops": fl}


def graph_us(dev, fns, reps=20):
    """µs per call of fns[i] (rotating), the calls captured once in a CUDA graph and replayed."""
    import torch
    s = torch.cuda.Stream(dev)
    with torch.cuda.stream(s):
        for f in fns:
            f()
        g = torch.cuda.CUDAGraph()
        g.capture_begin()
        for f in fns:
            f()
        g.capture_end()
        for _ in range(3):
            g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(reps):
            g.replay()
        e1.record(s)
    torch.cuda.synchronize(dev)
    del g
    return e0.elapsed_time(e1) / (reps * len(fns)) * 1e3


def measure_f16_packed(dw, dev, hbm):
    """fp16 I/O and packed batches (a NEXT row, outside the step) on the conformer workload,
    16x1500x512, K=9, lengths U[750,1500]: the forward in bf16 and in fp16 (same bytes), and the
    same sequences as a padded batch against a packed [N, C] batch (no padding rows), each over 3
    rotating input sets in a CUDA graph.  Algorithmic bytes: padded = x at valid frames + y in
    full; packed = x and y over the N valid rows."""
    import torch
    from synth import conv1d_inputs
    B, T, C, K, pl = 16, 1500, 512, 9, 4
    d = conv1d_inputs(B, T, C, K, dtype="f16", len_range=(750, 1500), seed=1)
    L = np.clip(d["lengths"], 0, T)
    w, bias = torch.from_numpy(d["w"]).to(dev), torch.from_numpy(d["bias"]).to(dev)
    ln = torch.from_numpy(d["lengths"]).to(dev)
    res = {}
    by_pad = (int(L.sum()) * C + B * T * C) * 2
    for name, td in (("padded_bf16", torch.bfloat16), ("padded_f16", torch.float16)):
        xs = [torch.from_numpy(d["x"]).to(dev, td) for _ in range(3)]
        ys = [torch.empty_like(xs[0]) for _ in range(3)]
        us = graph_us(dev, [lambda i=i: dw.dwconv1d_fwd(xs[i], w, bias, ys[i], ln, pl) for i in range(3)])
        res[name] = {"us": us, "GB_per_s": by_pad / us / 1e3, "hbm_frac_of_measured": by_pad / us / 1e3 / hbm,
                     "alg_bytes": by_pad}
        del xs, ys
    xp = np.concatenate([d["x"][b, :L[b]] for b in range(B)])
    N = xp.shape[0]
    offsets = torch.from_numpy(np.concatenate([[0], np.cumsum(L)]).astype(np.int32)).to(dev)
    by_pk = 2 * N * C * 2
    xs = [torch.from_numpy(xp).to(dev, torch.bfloat16) for _ in range(3)]
    ys = [torch.empty_like(xs[0]) for _ in range(3)]
    us = graph_us(dev, [lambda i=i: dw.dwconv1d_fwd_packed(xs[i], w, bias, ys[i], offsets, pl) for i in range(3)])
    res["packed_bf16"] = {"us": us, "GB_per_s": by_pk / us / 1e3, "hbm_frac_of_measured": by_pk / us / 1e3 / hbm,
                          "alg_bytes": by_pk, "rows": N, "padded_rows": B * T}
    # the weight gradient of the same packed batch (x and dy over the N rows read once)
    gw, gb = torch.empty(K, C, device=dev), torch.empty(C, device=dev)
    ws = torch.empty(dw.dwconv1d_bwd_dw_packed_workspace_size(B, N, C, K), dtype=torch.uint8, device=dev)
    us = graph_us(dev, [lambda i=i: dw.dwconv1d_bwd_dw_packed(xs[i], ys[i], gw, gb, offsets, pl, ws) for i in range(3)])
    res["packed_bf16_bwd_dw"] = {"us": us, "GB_per_s": by_pk / us / 1e3, "hbm_frac_of_measured": by_pk / us / 1e3 / hbm,
                                 "alg_bytes": by_pk}
    return {"workload": f"conformer dwconv1d forward {B}x{T}x{C}, K={K}, sym, len U[750,1500]: bf16 vs fp16 "
                        "padded, and the same sequences packed (3 rotating input sets in a CUDA graph)", **res}


def measure_batch_scaling(dw, dev, hbm):
    """The conv1d forward and dW on the conformer shape (T=1500, C=512, K=9, len U[750,1500]) at
    B = 16, 32 and 64 (a NEXT-row measurement, outside the step): graph replay over 3 rotating
    input sets.  Shows the fixed cost of a launch against the per-item cost, next to torch's
    elementwise kernel moving the forward's bytes (what a generic bandwidth-bound launch gets at
    each size)."""
    import torch
    from synth import conv1d_inputs
    T, C, K, pl = 1500, 512, 9, 4
    res = {}
    for B in (16, 32, 64):
        d = conv1d_inputs(B, T, C, K, dtype="bf16", len_range=(750, 1500), seed=1, with_dy=True)
        xs = [torch.from_numpy(d["x"]).to(dev, torch.bfloat16) for _ in range(3)]
        gs = [torch.from_numpy(d["dy"]).to(dev, torch.bfloat16) for _ in range(3)]
        ys = [torch.empty_like(xs[0]) for _ in range(3)]
        w, bias, ln = (torch.from_numpy(d["w"]).to(dev), torch.from_numpy(d["bias"]).to(dev),
                       torch.from_numpy(d["lengths"]).to(dev))
        gw, gb = torch.empty(K, C, device=dev), torch.empty(C, device=dev)
        ws = torch.empty(dw.dwconv1d_bwd_dw_workspace_size(B, T, C, K), dtype=torch.uint8, device=dev)
        L = np.clip(d["lengths"], 0, T)
        byf = (int(L.sum()) + B * T) * C * 2
        byw = 2 * int(L.sum()) * C * 2
        tf = graph_us(dev, [lambda i=i: dw.dwconv1d_fwd(xs[i], w, bias, ys[i], ln, pl) for i in range(3)])
        tw = graph_us(dev, [lambda i=i: dw.dwconv1d_bwd_dw(xs[i], gs[i], gw, gb, ln, pl, ws) for i in range(3)])
        # the floor at this size: torch's elementwise kernel (a STREAM-style scale, dst = 1 * src)
        # moving the forward's bytes, half read and half written, timed the same way
        srcs = [torch.zeros(byf // 4, dtype=torch.bfloat16, device=dev) for _ in range(3)]
        dsts = [torch.empty_like(srcs[0]) for _ in range(3)]
        tc = graph_us(dev, [lambda i=i: torch.mul(srcs[i], 1.0, out=dsts[i]) for i in range(3)])
        res[f"B{B}"] = {"fwd_us": tf, "fwd_hbm_frac_of_measured": byf / tf / 1e3 / hbm,
                        "dw_us": tw, "dw_hbm_frac_of_measured": byw / tw / 1e3 / hbm,
                        "copy_us": tc, "fwd_vs_copy": tc / tf}
        del xs, gs, ys, srcs, dsts
    return {"workload": f"conformer dwconv1d {T}x{C}, K={K}, bf16, len U[750,1500], B in 16/32/64 "
                        "(3 rotating input sets in a CUDA graph)", **res}


SWEEP = dict(B=32, T=750, C=1024, Ks=(3, 4, 5, 9, 15), odd=(520, 7), len_range=(375, 750), seed=2)


def measure_causal_sweep(dw, dev, hbm, fp32_tflops):
    """The causal kernel-width sweep: dwconv1d_fwd on x[32, 750, 1024] bf16 with K in {3,4,5,9,15},
    left padding K-1, lengths U[375,750], plus C=520, K=7 (channels not a multiple of 128); each over
    3 rotating input sets in a CUDA graph.  Algorithmic bytes: x at valid frames + y in full;
    flops 2K per valid output.  The roofline time is the larger of bytes / HBM and flops / FP32
    peak (K=15 comes near the balance); the max error is taken on items 0-1."""
    import torch
    import oracle
    from synth import conv1d_inputs
    c = SWEEP
    B, T = c["B"], c["T"]
    res = {}
    for C, K in [(c["C"], k) for k in c["Ks"]] + [c["odd"]]:
        d = conv1d_inputs(B, T, C, K, dtype="bf16", len_range=c["len_range"], seed=c["seed"])
        xs = [torch.from_numpy(d["x"]).to(dev, torch.bfloat16) for _ in range(3)]
        ys = [torch.empty_like(xs[0]) for _ in range(3)]
        w, bias, ln = (torch.from_numpy(d["w"]).to(dev), torch.from_numpy(d["bias"]).to(dev),
                       torch.from_numpy(d["lengths"]).to(dev))
        us = graph_us(dev, [lambda i=i: dw.dwconv1d_fwd(xs[i], w, bias, ys[i], ln, K - 1) for i in range(3)])
        valid = int(np.clip(d["lengths"], 0, T).sum())
        by = (valid + B * T) * C * 2 + (K + 1) * C * 4 + B * 4
        fl = 2 * K * valid * C
        t_roof = max(by / (hbm * 1e3), fl / (fp32_tflops * 1e6))  # µs
        dw.dwconv1d_fwd(xs[0], w, bias, ys[0], ln, K - 1)
        torch.cuda.synchronize(dev)
        got = ys[0][:2].float().cpu().numpy()
        ref = oracle.dwconv1d_fwd(d["x"][:2], d["w"], d["bias"], d["lengths"][:2], K - 1)
        res[f"C{C}_K{K}"] = {"us": us, "GB_per_s": by / us / 1e3, "frames_per_s": B * T / (us * 1e-6),
                             "hbm_frac_of_measured": by / us / 1e3 / hbm, "hbm_frac_of_8TBps": by / us / 1e3 / 8000.0,
                             "alu_frac": fl / us / 1e6 / fp32_tflops, "roofline_frac": t_roof / us,
                             "alg_bytes": by, "alg_flops": fl, "max_abs_err": float(np.max(np.abs(got - ref))),
                             "err_over_bar": bf16_err_over_bar(got, ref)}
        del xs, ys
    return {"workload": f"causal dwconv1d forward {B}x{T}x1024 bf16, K in {c['Ks']}, pads (K-1)|0, "
                        "len U[375,750]; plus C=520, K=7 (3 rotating input sets in a CUDA graph)", **res}


def measure_subsamplers(dw, dev, hbm, fp32_tflops):
    """The fused subsampler on mel[16, 3000, 80] -> [16, 750, 20, 256] bf16, len U[1500,3000]:
    symmetric and causal (time pad 2|0), through dw_subsample_fwd (conv0 on the tcgen05 tensor
    cores, the default) and dw_subsample_fwd_simt (every step on the FP32 pipes), each over 3
    rotating mel sets in a CUDA graph.  Algorithmic bytes: mel at valid frames + out in full;
    flops 18 per valid h element + 18 per valid output element.  fp32_frac is the roofline the
    depthwise path is stated against (the larger of bytes / HBM and flops / FP32 peak); for the
    tensor-core kernel, whose conv0 does not run on the FP32 pipes, the HBM fraction is the binding
    one.  The max error is taken on items 0-1."""
    import torch
    import oracle
    from synth import subsample_inputs
    B, T, F, C = SUB["B"], SUB["T"], SUB["F"], SUB["C"]
    ss = subsample_inputs(B, T, F, C, len_range=SUB["len_range"], seed=SUB["seed"])
    t = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    mels = [t(ss["mel"]) for _ in range(3)]
    w0, b0, w1, b1, ln = t(ss["w0"]), t(ss["b0"]), t(ss["w1"]), t(ss["b1"]), t(ss["lengths"], torch.int32)
    T4, F4 = dw.subsample_out_shape(T, F)
    outs = [torch.empty(B, T4, F4, C, dtype=torch.bfloat16, device=dev) for _ in range(3)]
    ol = torch.empty(B, dtype=torch.int32, device=dev)
    by, fl, _, _ = sub_work(ss["lengths"], T, F, C)
    res = {}
    for causal in (0, 1):
        ref, _ = oracle.dw_subsample_fwd(ss["mel"][:2], ss["w0"], ss["b0"], ss["w1"], ss["b1"], ss["lengths"][:2],
                                         causal)
        for name, fn in (("tc", dw.dw_subsample_fwd), ("fp32_simt", dw.dw_subsample_fwd_simt)):
            us = graph_us(dev, [lambda i=i: fn(mels[i], w0, b0, w1, b1, outs[i], ln, ol, causal) for i in range(3)])
            fn(mels[0], w0, b0, w1, b1, outs[0], ln, ol, causal)
            torch.cuda.synchronize(dev)
            got = outs[0][:2].float().cpu().numpy()
            t_fp32 = fl / (fp32_tflops * 1e6)
            t_hbm = by / (hbm * 1e3)
            r = {"us": us, "ms": us * 1e-3, "TFLOP_per_s": fl / us / 1e6, "fp32_frac": max(t_fp32, t_hbm) / us,
                 "hbm_frac_of_measured": t_hbm / us, "GB_per_s": by / us / 1e3,
                 "frames_per_s": B * T4 / (us * 1e-6), "alg_bytes": by, "alg_flops": fl,
                 "max_abs_err": float(np.max(np.abs(got - ref))), "err_over_bar": bf16_err_over_bar(got, ref)}
            if name == "tc":
                r["kernel"] = "dw_subsample_tc_kernel (conv0 on tcgen05, TF32 3-product split; ReLU, conv_dw1 on FP32)"
                r["roofline"] = "hbm"
            else:
                r["kernel"] = "dw_subsample_kernel (conv0, ReLU, conv_dw1 all packed FP32 FMA)"
                r["roofline"] = "fp32" if t_fp32 >= t_hbm else "hbm"
            res[f"{'causal' if causal else 'sym'}_{name}"] = r
    del mels, outs
    return {"workload": f"fused subsampler mel {B}x{T}x{F} fp32 -> {B}x{T4}x{F4}x{C} bf16, len U[1500,3000], "
                        "symmetric 1|1 and causal 2|0 (3 rotating mel sets in a CUDA graph)", **res}


CONV2D = dict(B=16, T=750, F=20, C=256, KT=3, KF=3, stride=(2, 2), pads=(1, 1, 1), len_range=(375, 750), seed=5)


def measure_conv2d(dw, dev, hbm):
    """General depthwise conv2d (a NEXT row, outside the step) on the subsampler's later-stage
    shape, [16, 750, 20, 256] bf16 -> [16, 375, 10, 256] with a 3x3 stride-2 window: forward, data
    gradient and weight/bias gradients, each over 3 rotating input sets in a CUDA graph.
    Algorithmic bytes: forward = x at valid frames + y in full; dx = dy at valid rows + dx in full;
    dW = x at valid frames + dy at valid rows."""
    import torch
    import oracle
    from synth import conv2d_inputs
    c = CONV2D
    B, T, F, C, KT, KF = c["B"], c["T"], c["F"], c["C"], c["KT"], c["KF"]
    stride, pads = c["stride"], c["pads"]
    To, Fo = dw.conv2d_out_shape(T, F, KT, KF, stride, pads)
    d = conv2d_inputs(B, T, F, C, KT, KF, dtype="bf16", len_range=c["len_range"], seed=c["seed"],
                      dy_shape=(B, To, Fo, C))
    x0 = torch.from_numpy(d["x"]).to(dev, torch.bfloat16)
    g0 = torch.from_numpy(d["dy"]).to(dev, torch.bfloat16)
    xs, gs = [x0] + [x0.clone() for _ in range(2)], [g0] + [g0.clone() for _ in range(2)]
    ys = [torch.empty(B, To, Fo, C, dtype=torch.bfloat16, device=dev) for _ in range(3)]
    dxs = [torch.empty_like(x0) for _ in range(3)]
    w = torch.from_numpy(d["w"]).to(dev)
    bias = torch.from_numpy(d["bias"]).to(dev)
    ln = torch.from_numpy(d["lengths"]).to(dev)
    ol = torch.empty(B, dtype=torch.int32, device=dev)
    gw, gb = torch.empty(KT, KF, C, device=dev), torch.empty(C, device=dev)
    ws = torch.empty(dw.dwconv2d_bwd_dw_workspace_size(B, T, F, C, KT, KF, stride, pads), dtype=torch.uint8,
                     device=dev)
    s = torch.cuda.Stream(dev)

    def timed(fn):
        with torch.cuda.stream(s):
            for i in range(3):
                fn(i)
            g = torch.cuda.CUDAGraph()
            g.capture_begin()
            for i in range(3):
                fn(i)
            g.capture_end()
            for _ in range(3):
                g.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            for _ in range(20):
                g.replay()
            e1.record(s)
        torch.cuda.synchronize(dev)
        del g
        return e0.elapsed_time(e1) / 60 * 1e3

    t_fwd = timed(lambda i: dw.dwconv2d_fwd(xs[i], w, bias, ys[i], ln, ol, stride, pads))
    t_dx = timed(lambda i: dw.dwconv2d_bwd_dx(gs[i], w, dxs[i], ln, stride, pads))
    t_dw = timed(lambda i: dw.dwconv2d_bwd_dw(xs[i], gs[i], gw, gb, ln, stride, pads, ws))
    L = np.clip(d["lengths"], 0, T)
    Lo = ol.cpu().numpy()  # output lengths as the forward reported them (checked against the oracle in tests)
    x_valid = int(L.sum()) * F * C * 2
    dy_valid = int(Lo.sum()) * Fo * C * 2
    by_fwd = x_valid + B * To * Fo * C * 2
    by_dx = dy_valid + B * T * F * C * 2
    by_dw = x_valid + dy_valid
    with torch.cuda.stream(s):
        dw.dwconv2d_fwd(xs[0], w, bias, ys[0], ln, ol, stride, pads)
    torch.cuda.synchronize(dev)
    ry, _ = oracle.dwconv2d_fwd(d["x"][:1], d["w"], d["bias"], d["lengths"][:1], stride, pads)
    err = float(np.max(np.abs(ys[0][:1].float().cpu().numpy() - ry)))

    def row(us, by):
        return {"us": us, "GB_per_s": by / us / 1e3, "hbm_frac_of_measured": by / us / 1e3 / hbm, "alg_bytes": by}
    return {"workload": f"depthwise conv2d {B}x{T}x{F}x{C} bf16 -> {B}x{To}x{Fo}x{C}, {KT}x{KF} stride 2, "
                        "pads 1|1|1, len U[375,750] (3 rotating input sets in a CUDA graph)",
            "fwd": row(t_fwd, by_fwd), "bwd_dx": row(t_dx, by_dx), "bwd_dw": row(t_dw, by_dw),
            "fwd_max_abs_err_item0": err}


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0}, "fallback"


def kernel_source_sha():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "speech_encoder_depthwise_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel):
    """Bytes per launch recorded from an ncu capture, if the kernels have not changed since:
    (DRAM bytes read + bytes the SMs wrote into L2, dram read, SM writes), else None."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        rows = [dict(kv.split("=", 1) for kv in line.split()) for line in open(path)
                if line.strip() and not line.startswith("#")]
    except Exception:
        return None
    sha = kernel_source_sha()
    for r in rows:
        if r.get("kernel") == kernel and r.get("sha") == sha:
            rd, wr = float(r["dram_read"]), float(r["sm_write"])
            return rd + wr, rd, wr
    return None


# ------------------------------------------------------------------ reference arm (CPU oracle)
def oracle_sample_step(cs, ss, frac):
    """One bounded oracle step: item 0 of each workload, the first `frac` of its frames."""
    import oracle
    Tc = max(CONV["K"], int(round(frac * CONV["T"])))
    Ts = max(8, 4 * int(round(frac * SUB["T"] / 4)))
    x, dy = cs["x"][:1, :Tc], cs["dy"][:1, :Tc]
    ln = np.minimum(cs["lengths"][:1], Tc).astype(np.int32)
    oracle.dwconv1d_fwd(x, cs["w"], cs["bias"], ln, CONV["pad_left"])
    oracle.dwconv1d_bwd_dx(dy, cs["w"], ln, CONV["pad_left"])
    oracle.dwconv1d_bwd_dw(x, dy, CONV["K"], ln, CONV["pad_left"])
    mel = ss["mel"][:1, :Ts]
    sl = np.minimum(ss["lengths"][:1], Ts).astype(np.int32)
    oracle.dw_subsample_fwd(mel, ss["w0"], ss["b0"], ss["w1"], ss["b1"], sl, SUB["causal"])
    w, _ = conv_work(ln, Tc, CONV["C"], CONV["K"])
    sb, _, _, _ = sub_work(sl, Ts, SUB["F"], SUB["C"])
    return sum(v[0] for v in w.values()) + sb, f"item 0, first {Tc} of {CONV['T']} conv1d frames and " \
        f"{Ts} of {SUB['T']} mel frames"


def inputs():
    from synth import conv1d_inputs, subsample_inputs
    cs = conv1d_inputs(CONV["B"], CONV["T"], CONV["C"], CONV["K"], dtype="bf16",
                       len_range=CONV["len_range"], seed=CONV["seed"], with_dy=True)
    ss = subsample_inputs(SUB["B"], SUB["T"], SUB["F"], SUB["C"], len_range=SUB["len_range"], seed=SUB["seed"])
    return cs, ss


def cpu_rate(cs, ss, seconds, steps=None):
    """Time the oracle on bounded samples; returns (GB/s, sample description, cores, per-step s)."""
    import oracle
    t0 = time.perf_counter()
    oracle_sample_step(cs, ss, 0.02)
    cal = max(time.perf_counter() - t0, 1e-3)
    per_step = seconds if steps is None else seconds / max(steps, 1)
    frac = float(min(1.0, max(0.01, 0.02 * per_step / cal)))
    total_b, total_t, n = 0, 0.0, 0
    desc = ""
    while True:
        t0 = time.perf_counter()
        b, desc = oracle_sample_step(cs, ss, frac)
        total_t += time.perf_counter() - t0
        total_b += b
        n += 1
        if steps is not None and n >= steps:
            break
        if steps is None and total_t >= seconds:
            break
    return total_b / total_t / 1e9, desc, oracle.num_threads(), total_t / n


def cpu_single_thread_cfg1_ms():
    """The oracle's conv1d forward on the fp32 parity workload (1x200x256, K=9, pads 4|4, no
    mask), on one host thread: median of 5 runs, in a subprocess with OMP_NUM_THREADS=1."""
    import subprocess
    code = ("import sys, time; sys.path.insert(0, %r)\n"
            "import numpy as np, oracle\n"
            "from synth import conv1d_inputs\n"
            "d = conv1d_inputs(1, 200, 256, 9, dtype='f32', len_range=None, seed=0)\n"
            "oracle.dwconv1d_fwd(d['x'], d['w'], d['bias'], None, 4)\n"
            "ts = []\n"
            "for _ in range(5):\n"
            "    t0 = time.perf_counter(); oracle.dwconv1d_fwd(d['x'], d['w'], d['bias'], None, 4)\n"
            "    ts.append(time.perf_counter() - t0)\n"
            "print(sorted(ts)[2] * 1e3, oracle.num_threads())\n") % ROOT
    try:
        r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120,
                           env=dict(os.environ, OMP_NUM_THREADS="1"))
        ms, thr = r.stdout.split()
        return {"ms": float(ms), "threads": int(thr), "workload": "conv1d forward 1x200x256 fp32, K=9, pads 4|4"}
    except Exception as e:  # reported, never fatal
        return {"unavailable": str(e)[:200]}


def reference_arm(args, world, rank):
    if rank != 0:
        return 0
    cs, ss = inputs()
    budget = 150.0  # seconds for warm-up + timed steps
    per = budget / (args.steps + max(args.warmup, 0))
    # warm-up steps (untimed)
    if args.warmup > 0:
        cpu_rate(cs, ss, per * args.warmup, steps=args.warmup)
    v, desc, cores, step_s = cpu_rate(cs, ss, per * args.steps, steps=args.steps)
    line = {"metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD, "parallelism": "rank 0 only (CPU)"},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def summary_table(line):
    """One compact string per kernel row (µs, roofline fraction, error / parity bar), placed last in
    the JSON line so that a reader of its tail sees every configuration."""
    out = {}

    def put(key, r, frac_key="hbm_frac_of_measured"):
        if r:
            out[key] = f"{r['us']:.1f}us {frac_key.split('_of')[0].replace('_frac', '')} {r[frac_key]:.2f}" + \
                (f" err/bar {r['err_over_bar']:.2f}" if "err_over_bar" in r else "")
    rows = line["rows"]
    put("cfg2_fwd", rows.get("dwconv1d_fwd"))
    put("cfg2_dx", rows.get("dwconv1d_bwd_dx"))
    put("cfg2_dw", rows.get("dwconv1d_bwd_dw"))
    cf = line.get("configs", {})
    for k, r in cf.get("causal_kernel_width_sweep", {}).items():
        if isinstance(r, dict):
            put(f"cfg3_{k}", r, "roofline_frac")
    for k, r in cf.get("subsampler", {}).items():
        if isinstance(r, dict):
            put(f"cfg4_{k}", r, "fp32_frac" if "simt" in k else "hbm_frac_of_measured")
    tb = cf.get("training_backward", {})
    put("cfg5_dx", tb.get("dwconv1d_bwd_dx"))
    put("cfg5_dw", tb.get("dwconv1d_bwd_dw"))
    put("cfg5_one_pass", tb.get("dwconv1d_bwd_one_pass"))
    return out


# ------------------------------------------------------------------ our arm
def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return reference_arm(args, world, rank)

    import torch
    import torch.distributed as dist
    import speech_encoder_depthwise_b200 as dw

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    lib = dw.lib()
    warmup = max(args.warmup, 3)
    steps = max(args.steps, 1)

    cs, ss = inputs()
    if rank > 0:  # each rank its own batch (weak scaling)
        from synth import conv1d_inputs, subsample_inputs
        cs = conv1d_inputs(CONV["B"], CONV["T"], CONV["C"], CONV["K"], dtype="bf16",
                           len_range=CONV["len_range"], seed=100 + rank, with_dy=True)
        ss = subsample_inputs(SUB["B"], SUB["T"], SUB["F"], SUB["C"], len_range=SUB["len_range"],
                              seed=200 + rank)
    B, T, C, K, pl = CONV["B"], CONV["T"], CONV["C"], CONV["K"], CONV["pad_left"]
    SB, ST, SF, SC = SUB["B"], SUB["T"], SUB["F"], SUB["C"]
    T4, F4 = dw.subsample_out_shape(ST, SF)

    def t(a, dtype=torch.float32):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev, dtype)

    w, bias, ln = t(cs["w"]), t(cs["bias"]), t(cs["lengths"], torch.int32)
    w0, b0, w1, b1, sl = t(ss["w0"]), t(ss["b0"]), t(ss["w1"]), t(ss["b1"]), t(ss["lengths"], torch.int32)
    x0, dy0, mel0 = t(cs["x"], torch.bfloat16), t(cs["dy"], torch.bfloat16), t(ss["mel"])
    sets = []
    for _ in range(N_SETS):
        sets.append(dict(x=x0.clone(), dy=dy0.clone(), y=torch.empty_like(x0), dx=torch.empty_like(x0),
                         mel=mel0.clone(), out=torch.empty(SB, T4, F4, SC, dtype=torch.bfloat16, device=dev)))
    del x0, dy0, mel0
    gw = torch.empty(K, C, device=dev)
    gb = torch.empty(C, device=dev)
    ol = torch.empty(SB, dtype=torch.int32, device=dev)
    nws = dw.dwconv1d_bwd_dw_workspace_size(B, T, C, K)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
    # the step runs on a side stream: it is captured into one CUDA graph per input set
    stream = torch.cuda.Stream(dev)
    sp = stream.cuda_stream
    P = lambda tt: ctypes.c_void_p(tt.data_ptr())

    # argument tuples built once: each launch is one foreign call, no tensor bookkeeping
    calls = []
    for s in sets:
        calls.append([
            ("dwconv1d_fwd", lib.dwconv1d_fwd, (P(s["x"]), P(w), P(bias), P(s["y"]), P(ln), B, T, C, K, pl,
                                                dw.DW_BF16, ctypes.c_void_p(sp))),
            ("dwconv1d_bwd_dx", lib.dwconv1d_bwd_dx, (P(s["dy"]), P(w), P(s["dx"]), P(ln), B, T, C, K, pl,
                                                      dw.DW_BF16, ctypes.c_void_p(sp))),
            ("dwconv1d_bwd_dw", lib.dwconv1d_bwd_dw, (P(s["x"]), P(s["dy"]), P(gw), P(gb), P(ln), B, T, C, K,
                                                      pl, dw.DW_BF16, P(ws), ws.numel(), ctypes.c_void_p(sp))),
            ("dw_subsample_fwd", lib.dw_subsample_fwd, (P(s["mel"]), P(w0), P(b0), P(w1), P(b1), P(s["out"]),
                                                        P(sl), P(ol), SB, ST, SF, SC, SUB["causal"],
                                                        dw.DW_BF16, ctypes.c_void_p(sp))),
        ])
    rows = [c[0] for c in calls[0]]
    launches_per_row = {"dwconv1d_fwd": 1, "dwconv1d_bwd_dx": 1, "dwconv1d_bwd_dw": 2, "dw_subsample_fwd": 1}

    def run_step(i, evs=None):
        for j, (name, fn, a) in enumerate(calls[i % N_SETS]):
            if evs is not None:
                evs[j][0].record(stream)
            st = fn(*a)
            if st != 0:
                raise RuntimeError(f"{name}: {dw.dw_status_string(st)}")
            if evs is not None:
                evs[j][1].record(stream)

    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for i in range(warmup):
            run_step(i)
        # one graph per input set: the 5 kernel launches of a step replayed without host work
        graphs = []
        for i in range(N_SETS):
            g = torch.cuda.CUDAGraph()
            g.capture_begin()
            run_step(i)
            g.capture_end()
            graphs.append(g)
        for i in range(warmup):
            graphs[i % N_SETS].replay()
    torch.cuda.synchronize(dev)

    mk = lambda: torch.cuda.Event(enable_timing=True)
    e_start, e_end = mk(), mk()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk, torch.cuda.stream(stream):
        e_start.record(stream)
        for i in range(steps):
            graphs[i % N_SETS].replay()
        e_end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    elapsed_ms = e_start.elapsed_time(e_end)
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    ms_per_step = elapsed_ms / steps

    # per-kernel durations (untimed above): each row's launches for the N_SETS input sets
    # captured in one CUDA graph and replayed back to back, as in the step; the eager figure
    # (each launch bracketed by events, launch gaps included) is kept beside it
    del graphs

    def row_graph_ms(j, reps=50):
        with torch.cuda.stream(stream):
            g = torch.cuda.CUDAGraph()
            g.capture_begin()
            for i in range(N_SETS):
                name, fn, a = calls[i][j]
                fn(*a)
            g.capture_end()
            for _ in range(3):
                g.replay()
            e0, e1 = mk(), mk()
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        del g
        return e0.elapsed_time(e1) / (reps * N_SETS)

    row_ms = {r: row_graph_ms(j) for j, r in enumerate(rows)}
    row_steps = min(steps, 200)
    step_evs = [[(mk(), mk()) for _ in rows] for _ in range(row_steps)]
    with torch.cuda.stream(stream):
        for i in range(row_steps):
            run_step(i, step_evs[i])
    torch.cuda.synchronize(dev)
    row_eager_ms = {r: float(np.mean([step_evs[i][j][0].elapsed_time(step_evs[i][j][1]) for i in range(row_steps)]))
                    for j, r in enumerate(rows)}

    cw, valid = conv_work(cs["lengths"], T, C, K)
    sb, sf, _, _ = sub_work(ss["lengths"], ST, SF, SC)
    step_bytes = sum(v[0] for v in cw.values()) + sb
    value = job_throughput(step_bytes, ms_per_step, world)

    # ---------------------------------------------------------------- e2e through the binding
    e2e = None
    if args.e2e_steps > 0:
        h = dict(x=torch.from_numpy(cs["x"]).to(torch.bfloat16).pin_memory(),
                 dy=torch.from_numpy(cs["dy"]).to(torch.bfloat16).pin_memory(),
                 ln=torch.from_numpy(cs["lengths"]).pin_memory(),
                 mel=torch.from_numpy(ss["mel"]).pin_memory(),
                 sl=torch.from_numpy(ss["lengths"]).pin_memory(),
                 w=torch.from_numpy(cs["w"]).pin_memory(), bias=torch.from_numpy(cs["bias"]).pin_memory(),
                 w0=torch.from_numpy(ss["w0"]).pin_memory(), b0=torch.from_numpy(ss["b0"]).pin_memory(),
                 w1=torch.from_numpy(ss["w1"]).pin_memory(), b1=torch.from_numpy(ss["b1"]).pin_memory())
        ho = dict(y=torch.empty(B, T, C, dtype=torch.bfloat16).pin_memory(),
                  dx=torch.empty(B, T, C, dtype=torch.bfloat16).pin_memory(),
                  gw=torch.empty(K, C).pin_memory(), gb=torch.empty(C).pin_memory(),
                  out=torch.empty(SB, T4, F4, SC, dtype=torch.bfloat16).pin_memory(),
                  ol=torch.empty(SB, dtype=torch.int32).pin_memory())
        h2d = sum(v.numel() * v.element_size() for v in h.values())
        d2h = sum(v.numel() * v.element_size() for v in ho.values())
        # Two device sets and three streams, as a serving pipeline runs: the inputs of step i go
        # up on s_in while step i-1 computes and step i-2's results come down on s_out (the two
        # copy directions use separate copy engines).  Set i % 2 is reused once step i-2's
        # results are down.  Every step still copies all of its inputs and outputs.
        dsets = []
        for k in range(2):
            z = sets[k]
            dsets.append(dict(x=z["x"], dy=z["dy"], y=z["y"], dx=z["dx"], mel=z["mel"], out=z["out"],
                              gw=torch.empty(K, C, device=dev), gb=torch.empty(C, device=dev),
                              ol=torch.empty(SB, dtype=torch.int32, device=dev),
                              w=torch.empty_like(w), bias=torch.empty_like(bias), w0=torch.empty_like(w0),
                              b0=torch.empty_like(b0), w1=torch.empty_like(w1), b1=torch.empty_like(b1),
                              ln=torch.empty_like(ln), sl=torch.empty_like(sl)))
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            k = i % 2
            z = dsets[k]
            if i >= 2:
                s_in.wait_event(ev_out[k])
            with torch.cuda.stream(s_in):
                for name in ("x", "dy", "mel", "w", "bias", "w0", "b0", "w1", "b1", "ln", "sl"):
                    z[name].copy_(h[name], non_blocking=True)
                ev_in[k].record(s_in)
            stream.wait_event(ev_in[k])
            with torch.cuda.stream(stream):  # the binding launches on the current stream
                dw.dwconv1d_fwd(z["x"], z["w"], z["bias"], z["y"], z["ln"], pl)
                dw.dwconv1d_bwd_dx(z["dy"], z["w"], z["dx"], z["ln"], pl)
                dw.dwconv1d_bwd_dw(z["x"], z["dy"], z["gw"], z["gb"], z["ln"], pl, ws)
                dw.dw_subsample_fwd(z["mel"], z["w0"], z["b0"], z["w1"], z["b1"], z["out"], z["sl"], z["ol"],
                                    SUB["causal"])
                ev_comp[k].record(stream)
            s_out.wait_event(ev_comp[k])
            with torch.cuda.stream(s_out):
                for name in ("y", "dx", "gw", "gb", "out", "ol"):
                    ho[name].copy_(z[name], non_blocking=True)
                ev_out[k].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        a, b_ = mk(), mk()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        a.record(s_in)
        for i in range(args.e2e_steps):
            e2e_step(i)
        s_in.wait_stream(s_out)
        b_.record(s_in)  # after the last step's results are down
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(a.elapsed_time(b_) / args.e2e_steps, world, dev)
        e2e = {"value": job_throughput(step_bytes, e2e_ms, world), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    # ---------------------------------------------------------------- report (rank 0)
    if rank == 0:
        peaks, peak_kind = measured_peaks()
        hbm = float(peaks.get("hbm_gbs", 6650.0))
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        fmax = float(peaks.get("sm_max_mhz", 1965.0))
        fp32_tflops = sms * 128 * 2 * fmax * 1e6 / 1e12
        row = {}
        for name, (by, fl) in cw.items():
            key = {"fwd": "dwconv1d_fwd", "dx": "dwconv1d_bwd_dx", "dw": "dwconv1d_bwd_dw"}[name]
            ms = row_ms[key]
            row[key] = {"us": ms * 1e3, "eager_us": row_eager_ms[key] * 1e3, "GB_per_s": by / (ms * 1e-3) / 1e9,
                        "frames_per_s": B * T / (ms * 1e-3),
                        "hbm_frac_of_measured": by / (ms * 1e-3) / 1e9 / hbm,
                        "hbm_frac_of_8TBps": by / (ms * 1e-3) / 1e9 / 8000.0,
                        "alg_bytes": by, "alg_flops": fl}
        ms = row_ms["dw_subsample_fwd"]
        row["dw_subsample_fwd"] = {"kernel": "dw_subsample_tc_kernel (conv0 on tcgen05)",
                                   "ms": ms, "us": ms * 1e3, "eager_us": row_eager_ms["dw_subsample_fwd"] * 1e3,
                                   "TFLOP_per_s": sf / (ms * 1e-3) / 1e12,
                                   "hbm_frac_of_measured": sb / (ms * 1e-3) / 1e9 / hbm,
                                   "fp32_term_frac": sf / (ms * 1e-3) / 1e12 / fp32_tflops,
                                   "GB_per_s": sb / (ms * 1e-3) / 1e9,
                                   "frames_per_s": SB * T4 / (ms * 1e-3),
                                   "alg_bytes": sb, "alg_flops": sf}
        # every throughput row carries its distance from the oracle (items 0-1; dW over the batch)
        import oracle
        f64 = lambda tt: tt.float().cpu().numpy().astype(np.float64)
        s0 = sets[0]
        err = lambda a, b: float(np.max(np.abs(a - b)))
        ry = oracle.dwconv1d_fwd(cs["x"][:2], cs["w"], cs["bias"], cs["lengths"][:2], pl)
        row["dwconv1d_fwd"]["max_abs_err"] = err(f64(s0["y"][:2]), ry)
        row["dwconv1d_fwd"]["err_over_bar"] = bf16_err_over_bar(f64(s0["y"][:2]), ry)
        rdx = oracle.dwconv1d_bwd_dx(cs["dy"][:2], cs["w"], cs["lengths"][:2], pl)
        row["dwconv1d_bwd_dx"]["max_abs_err"] = err(f64(s0["dx"][:2]), rdx)
        row["dwconv1d_bwd_dx"]["err_over_bar"] = bf16_err_over_bar(f64(s0["dx"][:2]), rdx)
        rdw, rdb = oracle.dwconv1d_bwd_dw(cs["x"], cs["dy"], K, cs["lengths"], pl)
        row["dwconv1d_bwd_dw"]["max_abs_err"] = max(err(f64(gw), rdw), err(f64(gb), rdb))
        row["dwconv1d_bwd_dw"]["err_over_bar"] = max(dw_err_over_bar(f64(gw), rdw), dw_err_over_bar(f64(gb), rdb))
        ro, _ = oracle.dw_subsample_fwd(ss["mel"][:2], ss["w0"], ss["b0"], ss["w1"], ss["b1"],
                                        ss["lengths"][:2], SUB["causal"])
        row["dw_subsample_fwd"]["max_abs_err"] = err(f64(s0["out"][:2]), ro)
        row["dw_subsample_fwd"]["err_over_bar"] = bf16_err_over_bar(f64(s0["out"][:2]), ro)
        want = {"sweep", "sub", "bwd", "stream", "conv2d", "f16_packed", "sub_bwd", "batch"} \
            if args.next_rows == "all" else set() if args.next_rows == "none" else set(args.next_rows.split(","))
        cfg_measures = [("sweep", "causal_kernel_width_sweep", lambda: measure_causal_sweep(dw, dev, hbm, fp32_tflops)),
                        ("sub", "subsampler", lambda: measure_subsamplers(dw, dev, hbm, fp32_tflops)),
                        ("bwd", "training_backward", lambda: measure_bwd(dw, dev, hbm))]
        measures = [("stream", "dwconv1d_stream_fwd", lambda: measure_stream(dw, dev, hbm)),
                    ("conv2d", "dwconv2d", lambda: measure_conv2d(dw, dev, hbm)),
                    ("f16_packed", "f16_and_packed", lambda: measure_f16_packed(dw, dev, hbm)),
                    ("sub_bwd", "dw_subsample_bwd", lambda: measure_sub_bwd(dw, dev, hbm, fp32_tflops)),
                    ("batch", "conv1d_batch_scaling", lambda: measure_batch_scaling(dw, dev, hbm))]
        with ClockSampler(local) as clk_rows:
            configs = {name: fn() for key, name, fn in cfg_measures if key in want}
            next_rows = {name: fn() for key, name, fn in measures if key in want}
        cpu = None
        if world == 1 and args.cpu_seconds > 0:
            v, desc, cores, _ = cpu_rate(cs, ss, args.cpu_seconds)
            cpu = {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc,
                   "single_thread_cfg1": cpu_single_thread_cfg1_ms()}
        clocks = clk.summary()
        if clk_rows.samples:  # the timed steps are ~2 ms: add the samples of the per-config replays
            clocks = dict(clocks, window="timed steps and the per-config graph replays after them",
                          sm_mhz=float(np.median(clk.samples + clk_rows.samples)),
                          reasons=sorted(set(clocks["reasons"]) | clk_rows.reasons),
                          samples=len(clk.samples) + len(clk_rows.samples))
        simt = configs.get("subsampler", {}).get("sym_fp32_simt")
        tc_traffic = ncu_traffic("dw_subsample_tc_kernel")
        tc_us = ms * 1e3
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": steps,
            "warmup": warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; shapes of the pages' workloads)",
            "config": {"workload": WORKLOAD, "global_batch": world * B, "seq_len": T,
                       "parallelism": f"replicas x{world} (independent batches, no collective)",
                       "l2": f"{N_SETS} rotating input sets of ~237 MB each (> L2 126 MB)"},
            "frames_per_s": world * B * T / (row_ms["dwconv1d_fwd"] * 1e-3),
            # the depthwise subsampler metric on the all-FP32 kernel (its roofline: max(bytes / HBM,
            # flops / FP32 peak)); the tensor-core kernel the step runs is reported beside it
            "subsampler_ms": simt["ms"] if simt else None,
            "subsampler_roofline_frac": simt["fp32_frac"] if simt else None,
            "subsampler_fp32_pipe_frac": simt["TFLOP_per_s"] / fp32_tflops if simt else None,
            "subsampler_tc_ms": ms, "subsampler_tc_hbm_frac": sb / (ms * 1e-3) / 1e9 / hbm,
            "rows": row,
            "configs": configs,
            "roofline": {"bound": "hbm", "kernel": "dw_subsample_tc_kernel",
                         "achieved": sb / (ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                         "frac": sb / (ms * 1e-3) / 1e9 / hbm,
                         "traffic": tc_traffic[0] if tc_traffic else None,
                         "traffic_split": {"dram_read": tc_traffic[1], "sm_write_to_l2": tc_traffic[2],
                                           "method": "ncu dram__bytes_read.sum + 32 x "
                                                     "lts__t_sectors_srcunit_tex_op_write.sum, one launch"}
                         if tc_traffic else None,
                         "peak_kind": f"{peak_kind} HBM copy bandwidth",
                         "note": "the step's dominant kernel, bound by HBM on the resources it uses: conv0 runs on "
                                 "tcgen05 (TF32 3-product split), ReLU and conv_dw1 on the FP32 pipes "
                                 f"({sf / 1e9:.2f} GFLOP algorithmic, {sf / tc_us / 1e6 / fp32_tflops:.2f} of the "
                                 f"FP32 peak {fp32_tflops:.1f} TFLOP/s = {sms} SMs x 128 x 2 x {fmax:.0f} MHz)"},
            "hbm_peak_gbs": hbm, "hbm_peak_kind": peak_kind,
            "cpu_baseline": cpu, "e2e": e2e,
            "next_rows": next_rows,
            "gpu_launches": steps * sum(launches_per_row.values()),
            "clocks": clocks,
        }
        line["summary"] = summary_table(line)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
