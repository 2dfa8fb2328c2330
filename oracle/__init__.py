"""CPU oracle for the depthwise-convolution hot path (fp64, plain loops).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU baseline
import this package.  The product path (the CUDA library and its Python binding) never
imports it, and it imports nothing from the product.

The arithmetic lives in ``dwconv_oracle.c`` (compiled here with gcc into
``oracle/_build/liboracle.so``); this module only compiles it, converts numpy arrays to
float64 and calls it.  Every function follows the definitions stated in that file, taken
from parakeet.cpp PR #102 ("What changes": the depthwise conv as a sum over the padded
input) and NeMo PR #16114 ("What does this PR do ?": conv0 -> ReLU -> masking -> conv_dw1,
with pre/post masking and causal padding).

Parity is pinned by ``tests/test_oracle_pins.py`` (a second formulation by im2col + matmul,
torch's float64 CPU convolutions, hand-worked golden values and invariants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dwconv_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()

_D = ctypes.POINTER(ctypes.c_double)
_I = ctypes.POINTER(ctypes.c_int32)
_L = ctypes.c_int64


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle with gcc (-O2, strict IEEE: no fast-math, no FMA contraction) and OpenMP."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", "-o", tmp, src]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _dp(a):
    return a.ctypes.data_as(_D) if a is not None else None


def _ip(a):
    return a.ctypes.data_as(_I) if a is not None else None


def _lens(lengths, B):
    if lengths is None:
        return None
    a = np.ascontiguousarray(lengths, dtype=np.int32)
    if a.shape != (B,):
        raise ValueError("lengths must have shape [B]")
    return a


def subsample_out_shape(T, F, causal):
    """(T4, F4) of the two stride-2 stages (time pads 1|1 or 2|0, frequency pads 1|1)."""
    def s2(n):
        return (n + 2 - 3) // 2 + 1 if n >= 1 else 0
    return s2(s2(T)), s2(s2(F))


class Oracle:
    """The oracle's functions, bound to one compiled copy of ``dwconv_oracle.c``."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_dwconv1d_fwd.argtypes = [_D, _D, _D, _I, _L, _L, _L, _L, _L, _D]
        lib.oracle_dwconv1d_bwd_dx.argtypes = [_D, _D, _I, _L, _L, _L, _L, _L, _D]
        lib.oracle_dwconv1d_bwd_dw.argtypes = [_D, _D, _I, _L, _L, _L, _L, _L, _D, _D]
        lib.oracle_dw_subsample_fwd.argtypes = [_D, _D, _D, _D, _D, _I, _L, _L, _L, _L,
                                                ctypes.c_int, _D, _I]
        lib.oracle_dwconv1d_stream_fwd.argtypes = [_D, _D, _D, _D, _I, _L, _L, _L, _L, _D, _D]
        lib.oracle_dw_subsample_bwd.argtypes = [_D, _D, _D, _D, _D, _I, _L, _L, _L, _L, ctypes.c_int,
                                                _D, _D, _D, _D]
        lib.oracle_dw_subsample_bwd_kinks.argtypes = [_D, _D, _D, _D, _D, _I, _L, _L, _L, _L, ctypes.c_int,
                                                      ctypes.c_double, ctypes.c_double, _D, _D]
        lib.oracle_dwconv2d_fwd.argtypes = [_D, _D, _D, _I] + [_L] * 11 + [_D, _I]
        lib.oracle_dwconv2d_bwd_dx.argtypes = [_D, _D, _I] + [_L] * 11 + [_D]
        lib.oracle_dwconv2d_bwd_dw.argtypes = [_D, _D, _I] + [_L] * 11 + [_D, _D]
        for f in ("oracle_dwconv1d_fwd", "oracle_dwconv1d_bwd_dx", "oracle_dwconv1d_bwd_dw",
                  "oracle_dw_subsample_fwd", "oracle_dwconv1d_stream_fwd", "oracle_dw_subsample_bwd",
                  "oracle_dw_subsample_bwd_kinks", "oracle_dwconv2d_fwd", "oracle_dwconv2d_bwd_dx",
                  "oracle_dwconv2d_bwd_dw"):
            getattr(lib, f).restype = ctypes.c_int
        self.lib = lib
        self.path = lib_path

    def num_threads(self) -> int:
        """OpenMP threads the oracle runs with."""
        return int(self.lib.oracle_num_threads())

    def dwconv1d_fwd(self, x, w, bias, lengths, pad_left):
        """y[b,t,c] = [t<len_b] (bias[c] + sum_k xpad[b,t+k,c] w[k,c]); x [B,T,C], w [K,C]."""
        x = _f64(x); w = _f64(w)
        B, T, C = x.shape
        K = w.shape[0]
        assert w.shape == (K, C)
        b = _f64(bias) if bias is not None else None
        ln = _lens(lengths, B)
        y = np.empty((B, T, C), dtype=np.float64)
        rc = self.lib.oracle_dwconv1d_fwd(_dp(x), _dp(w), _dp(b), _ip(ln),
                                          B, T, C, K, int(pad_left), _dp(y))
        if rc:
            raise ValueError(f"oracle_dwconv1d_fwd rejected its arguments (rc={rc})")
        return y

    def dwconv1d_stream_fwd(self, x, w, bias, cache, lengths):
        """One chunk of the streaming causal conv: returns (y [B,T,C], new cache [B,K-1,C]).

        cache [B,K-1,C] holds each stream's K-1 most recent frames; the chunk appends the first
        lengths[b] frames of x[b] (all T when lengths is None)."""
        x = _f64(x); w = _f64(w)
        B, T, C = x.shape
        K = w.shape[0]
        assert w.shape == (K, C)
        cin = _f64(cache) if K > 1 else np.zeros((B, 0, C))
        assert cin.shape == (B, K - 1, C)
        b = _f64(bias) if bias is not None else None
        ln = _lens(lengths, B)
        y = np.empty((B, T, C), dtype=np.float64)
        cout = np.empty((B, K - 1, C), dtype=np.float64)
        rc = self.lib.oracle_dwconv1d_stream_fwd(_dp(x), _dp(w), _dp(b), _dp(cin) if K > 1 else None,
                                                 _ip(ln), B, T, C, K, _dp(y), _dp(cout) if K > 1 else None)
        if rc:
            raise ValueError(f"oracle_dwconv1d_stream_fwd rejected its arguments (rc={rc})")
        return y, cout

    def dwconv1d_bwd_dx(self, dy, w, lengths, pad_left):
        """Data gradient of ``dwconv1d_fwd`` (the transpose of the forward map)."""
        dy = _f64(dy); w = _f64(w)
        B, T, C = dy.shape
        K = w.shape[0]
        assert w.shape == (K, C)
        ln = _lens(lengths, B)
        dx = np.empty((B, T, C), dtype=np.float64)
        rc = self.lib.oracle_dwconv1d_bwd_dx(_dp(dy), _dp(w), _ip(ln),
                                             B, T, C, K, int(pad_left), _dp(dx))
        if rc:
            raise ValueError(f"oracle_dwconv1d_bwd_dx rejected its arguments (rc={rc})")
        return dx

    def dwconv1d_bwd_dw(self, x, dy, K, lengths, pad_left):
        """Weight and bias gradients: returns (dW [K,C], dbias [C])."""
        x = _f64(x); dy = _f64(dy)
        B, T, C = x.shape
        assert dy.shape == x.shape
        ln = _lens(lengths, B)
        dw = np.empty((int(K), C), dtype=np.float64)
        db = np.empty((C,), dtype=np.float64)
        rc = self.lib.oracle_dwconv1d_bwd_dw(_dp(x), _dp(dy), _ip(ln),
                                             B, T, C, int(K), int(pad_left), _dp(dw), _dp(db))
        if rc:
            raise ValueError(f"oracle_dwconv1d_bwd_dw rejected its arguments (rc={rc})")
        return dw, db

    def dw_subsample_fwd(self, mel, w0, b0, w1, b1, lengths, causal):
        """Fused subsampler front in fp64: returns (out [B,T4,F4,C], out_lengths [B])."""
        mel = _f64(mel)
        B, T, F = mel.shape
        w0 = _f64(w0); w1 = _f64(w1); b0 = _f64(b0); b1 = _f64(b1)
        C = w0.shape[-1]
        assert w0.shape == (3, 3, C) and w1.shape == (3, 3, C)
        assert b0.shape == (C,) and b1.shape == (C,)
        T4, F4 = subsample_out_shape(T, F, causal)
        ln = _lens(lengths, B)
        out = np.empty((B, T4, F4, C), dtype=np.float64)
        ol = np.empty((B,), dtype=np.int32)
        rc = self.lib.oracle_dw_subsample_fwd(_dp(mel), _dp(w0), _dp(b0), _dp(w1), _dp(b1),
                                              _ip(ln), B, T, F, C, int(bool(causal)),
                                              _dp(out), _ip(ol))
        if rc:
            raise ValueError(f"oracle_dw_subsample_fwd rejected its arguments (rc={rc})")
        return out, ol

    def dw_subsample_bwd(self, mel, w0, b0, w1, dout, lengths, causal):
        """Gradients of sum(out * dout) of the fused subsampler with respect to w0, b0, w1 and b1:
        returns (dw0 [3,3,C], db0 [C], dw1 [3,3,C], db1 [C])."""
        mel = _f64(mel); w0 = _f64(w0); b0 = _f64(b0); w1 = _f64(w1); dout = _f64(dout)
        B, T, F = mel.shape
        C = w0.shape[-1]
        T4, F4 = subsample_out_shape(T, F, causal)
        assert dout.shape == (B, T4, F4, C)
        ln = _lens(lengths, B)
        dw0 = np.empty((3, 3, C)); db0 = np.empty(C); dw1 = np.empty((3, 3, C)); db1 = np.empty(C)
        rc = self.lib.oracle_dw_subsample_bwd(_dp(mel), _dp(w0), _dp(b0), _dp(w1), _dp(dout), _ip(ln),
                                              B, T, F, C, int(bool(causal)), _dp(dw0), _dp(db0),
                                              _dp(dw1), _dp(db1))
        if rc:
            raise ValueError(f"oracle_dw_subsample_bwd rejected its arguments (rc={rc})")
        return dw0, db0, dw1, db1

    def dw_subsample_bwd_kinks(self, mel, w0, b0, w1, dout, lengths, causal, delta, delta_rel=0.0):
        """Bounds on how much dw0 / db0 can move when the ReLU decision flips at h pixels with
        |z| <= delta + delta_rel * S, S = |b0| + sum_t |melpad_t w0_t| (the magnitudes of z's
        terms): returns (kdw0 [3,3,C], kdb0 [C])."""
        mel = _f64(mel); w0 = _f64(w0); b0 = _f64(b0); w1 = _f64(w1); dout = _f64(dout)
        B, T, F = mel.shape
        C = w0.shape[-1]
        ln = _lens(lengths, B)
        kdw0 = np.empty((3, 3, C)); kdb0 = np.empty(C)
        rc = self.lib.oracle_dw_subsample_bwd_kinks(_dp(mel), _dp(w0), _dp(b0), _dp(w1), _dp(dout), _ip(ln),
                                                    B, T, F, C, int(bool(causal)), float(delta),
                                                    float(delta_rel), _dp(kdw0), _dp(kdb0))
        if rc:
            raise ValueError(f"oracle_dw_subsample_bwd_kinks rejected its arguments (rc={rc})")
        return kdw0, kdb0

    def dwconv2d_fwd(self, x, w, bias, lengths, stride, pads):
        """Depthwise conv2d, channels-last x [B,T,F,C], w [KT,KF,C]; stride (st, sf), pads (pt, pb, pf).
        Returns (y [B,To,Fo,C], out_lengths [B])."""
        x = _f64(x); w = _f64(w)
        B, T, F, C = x.shape
        KT, KF = w.shape[:2]
        (st, sf), (pt, pb, pf) = stride, pads
        To, Fo = conv2d_out_shape(T, F, KT, KF, stride, pads)
        b = _f64(bias) if bias is not None else None
        ln = _lens(lengths, B)
        y = np.empty((B, To, Fo, C)); ol = np.empty(B, dtype=np.int32)
        rc = self.lib.oracle_dwconv2d_fwd(_dp(x), _dp(w), _dp(b), _ip(ln), B, T, F, C, KT, KF, st, sf, pt, pb, pf,
                                          _dp(y), _ip(ol))
        if rc:
            raise ValueError(f"oracle_dwconv2d_fwd rejected its arguments (rc={rc})")
        return y, ol

    def dwconv2d_bwd_dx(self, dy, w, lengths, T, F, stride, pads):
        """Data gradient of dwconv2d_fwd: dx [B,T,F,C] from dy [B,To,Fo,C]."""
        dy = _f64(dy); w = _f64(w)
        B, To, Fo, C = dy.shape
        KT, KF = w.shape[:2]
        (st, sf), (pt, pb, pf) = stride, pads
        assert (To, Fo) == conv2d_out_shape(T, F, KT, KF, stride, pads)
        ln = _lens(lengths, B)
        dx = np.empty((B, T, F, C))
        rc = self.lib.oracle_dwconv2d_bwd_dx(_dp(dy), _dp(w), _ip(ln), B, T, F, C, KT, KF, st, sf, pt, pb, pf, _dp(dx))
        if rc:
            raise ValueError(f"oracle_dwconv2d_bwd_dx rejected its arguments (rc={rc})")
        return dx

    def dwconv2d_bwd_dw(self, x, dy, KT, KF, lengths, stride, pads):
        """Weight and bias gradients of dwconv2d_fwd: returns (dW [KT,KF,C], dbias [C])."""
        x = _f64(x); dy = _f64(dy)
        B, T, F, C = x.shape
        (st, sf), (pt, pb, pf) = stride, pads
        assert dy.shape[1:3] == conv2d_out_shape(T, F, KT, KF, stride, pads)
        ln = _lens(lengths, B)
        dw = np.empty((KT, KF, C)); db = np.empty(C)
        rc = self.lib.oracle_dwconv2d_bwd_dw(_dp(x), _dp(dy), _ip(ln), B, T, F, C, KT, KF, st, sf, pt, pb, pf,
                                             _dp(dw), _dp(db))
        if rc:
            raise ValueError(f"oracle_dwconv2d_bwd_dw rejected its arguments (rc={rc})")
        return dw, db


def conv2d_out_shape(T, F, KT, KF, stride, pads):
    """(To, Fo) of dwconv2d_fwd: (n + pads - k) // s + 1 per axis, 0 when the window does not fit."""
    (st, sf), (pt, pb, pf) = stride, pads
    def o(n, p0, p1, k, s):
        m = n + p0 + p1 - k
        return 0 if m < 0 else m // s + 1
    return o(T, pt, pb, KT, st), o(F, pf, pf, KF, sf)


def default() -> Oracle:
    """The oracle compiled from this package's source (built on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


_default = None


def num_threads() -> int:
    return default().num_threads()


def dwconv1d_fwd(x, w, bias, lengths, pad_left):
    return default().dwconv1d_fwd(x, w, bias, lengths, pad_left)


def dwconv1d_stream_fwd(x, w, bias, cache, lengths):
    return default().dwconv1d_stream_fwd(x, w, bias, cache, lengths)


def dwconv1d_fwd_packed(x, w, bias, offsets, pad_left):
    """A packed batch ("GPU inference for speech", section "Where the time goes": packed
    sequences instead of padding): x [N, C] holds the sequences back to back, sequence b on rows
    offsets[b]:offsets[b+1].  Each one is convolved on its own by ``dwconv1d_fwd`` (one item, its
    own length, no padding rows).  Rows no sequence covers come back as NaN."""
    x = np.asarray(x, np.float64)
    y = np.full(x.shape, np.nan)
    for b in range(len(offsets) - 1):
        s0, e = int(offsets[b]), int(offsets[b + 1])
        if e > s0:
            y[s0:e] = dwconv1d_fwd(x[None, s0:e], w, bias, None, pad_left)[0]
    return y


def dwconv1d_bwd_dw_packed(x, dy, K, offsets, pad_left):
    """Weight and bias gradients of ``dwconv1d_fwd_packed``: ``dwconv1d_bwd_dw`` of every sequence,
    summed.  Returns (dW [K, C], dbias [C])."""
    x = np.asarray(x, np.float64)
    dy = np.asarray(dy, np.float64)
    C = x.shape[1]
    gw, gb = np.zeros((K, C)), np.zeros(C)
    for b in range(len(offsets) - 1):
        s0, e = int(offsets[b]), int(offsets[b + 1])
        if e > s0:
            w_b, b_b = dwconv1d_bwd_dw(x[None, s0:e], dy[None, s0:e], K, None, pad_left)
            gw += w_b
            gb += b_b
    return gw, gb


def dwconv1d_bwd_dx_packed(dy, w, offsets, pad_left):
    """Data gradient of ``dwconv1d_fwd_packed``: ``dwconv1d_bwd_dx`` sequence by sequence."""
    dy = np.asarray(dy, np.float64)
    dx = np.full(dy.shape, np.nan)
    for b in range(len(offsets) - 1):
        s0, e = int(offsets[b]), int(offsets[b + 1])
        if e > s0:
            dx[s0:e] = dwconv1d_bwd_dx(dy[None, s0:e], w, None, pad_left)[0]
    return dx


def dw_subsample_bwd(mel, w0, b0, w1, dout, lengths, causal):
    return default().dw_subsample_bwd(mel, w0, b0, w1, dout, lengths, causal)


def dw_subsample_bwd_kinks(mel, w0, b0, w1, dout, lengths, causal, delta, delta_rel=0.0):
    return default().dw_subsample_bwd_kinks(mel, w0, b0, w1, dout, lengths, causal, delta, delta_rel)


def dwconv1d_bwd_dx(dy, w, lengths, pad_left):
    return default().dwconv1d_bwd_dx(dy, w, lengths, pad_left)


def dwconv1d_bwd_dw(x, dy, K, lengths, pad_left):
    return default().dwconv1d_bwd_dw(x, dy, K, lengths, pad_left)


def dw_subsample_fwd(mel, w0, b0, w1, b1, lengths, causal):
    return default().dw_subsample_fwd(mel, w0, b0, w1, b1, lengths, causal)


def dwconv2d_fwd(x, w, bias, lengths, stride, pads):
    return default().dwconv2d_fwd(x, w, bias, lengths, stride, pads)


def dwconv2d_bwd_dx(dy, w, lengths, T, F, stride, pads):
    return default().dwconv2d_bwd_dx(dy, w, lengths, T, F, stride, pads)


def dwconv2d_bwd_dw(x, dy, KT, KF, lengths, stride, pads):
    return default().dwconv2d_bwd_dw(x, dy, KT, KF, lengths, stride, pads)
