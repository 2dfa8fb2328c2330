"""B200 (sm_100a) depthwise-convolution hot path of a conformer speech encoder.

A thin binding over the C ABI of ``libdwconv_b200.so`` (declared in ``include/dwconv.h``):
each function below has the name of the C entry point it calls and only marshals arguments
(device pointers, sizes, dtype, the current CUDA stream).  Every step of the computation
runs in the library's CUDA kernels; there is no other code path.  If the library is missing,
every call raises: build it with ``python -m speech_encoder_depthwise_b200.build``.

Tensors are torch CUDA tensors, contiguous, channels last:
x, y, dy, dx ``[B, T, C]`` (bfloat16, float16 or float32); w ``[K, C]`` float32; bias ``[C]`` float32;
lengths ``[B]`` int32 (or None); mel ``[B, T, F]`` float32; w0, w1 ``[3, 3, C]`` float32.
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "DW_OK", "DW_ERR_INVALID_ARG", "DW_ERR_UNSUPPORTED", "DW_ERR_WORKSPACE", "DW_ERR_CUDA",
    "DW_ERR_TIMEOUT", "DW_F32", "DW_BF16", "DW_F16", "DwError", "lib", "library_path",
    "dwconv1d_fwd", "dwconv1d_bwd_dx", "dwconv1d_bwd_dw_workspace_size", "dwconv1d_bwd_dw",
    "dwconv1d_bwd_dw_noalloc", "dwconv1d_bwd", "dwconv1d_stream_fwd", "dwconv1d_fwd_packed",
    "dwconv1d_bwd_dx_packed", "dwconv1d_bwd_dw_packed_workspace_size", "dwconv1d_bwd_dw_packed",
    "dw_subsample_fwd", "dw_subsample_fwd_simt", "dw_subsample_bwd_workspace_size", "dw_subsample_bwd", "dw_status_string", "dw_device_error", "subsample_out_shape",
    "dwconv2d_fwd", "dwconv2d_bwd_dx", "dwconv2d_bwd_dw_workspace_size", "dwconv2d_bwd_dw", "conv2d_out_shape",
    "dw_selftest_wait_timeout",
]

DW_OK, DW_ERR_INVALID_ARG, DW_ERR_UNSUPPORTED, DW_ERR_WORKSPACE, DW_ERR_CUDA, DW_ERR_TIMEOUT = range(6)
DW_F32, DW_BF16, DW_F16 = 0, 1, 2

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libdwconv_b200.so")
_lock = threading.Lock()
_lib = None

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int

# name -> (restype, argtypes), mirroring include/dwconv.h
SIGNATURES = {
    "dwconv1d_fwd": (_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _int, _int, _vp]),
    "dwconv1d_bwd_dx": (_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _int, _int, _vp]),
    "dwconv1d_bwd_dw_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64, _int]),
    "dwconv1d_bwd_dw": (_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _int, _int, _vp,
                               ctypes.c_size_t, _vp]),
    "dwconv1d_bwd_dw_noalloc": (_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _int, _int, _vp]),
    "dwconv1d_bwd": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _int, _int, _vp,
                            ctypes.c_size_t, _vp]),
    "dwconv1d_stream_fwd": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _int, _vp]),
    "dwconv1d_fwd_packed": (_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _int, _int, _vp]),
    "dwconv1d_bwd_dx_packed": (_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _int, _int, _vp]),
    "dwconv1d_bwd_dw_packed_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64, _int]),
    "dwconv1d_bwd_dw_packed": (_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _int, _int, _vp,
                                      ctypes.c_size_t, _vp]),
    "dw_subsample_fwd": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                _int, _int, _vp]),
    "dw_subsample_fwd_simt": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                     _int, _int, _vp]),
    "dw_subsample_bwd_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64, _i64]),
    "dw_subsample_bwd": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _int,
                                _int, _vp, ctypes.c_size_t, _vp]),
    "dwconv2d_fwd": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _int, _int, _int, _int, _int,
                            _int, _int, _int, _vp]),
    "dwconv2d_bwd_dx": (_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _int, _int, _int, _int, _int, _int,
                               _int, _int, _vp]),
    "dwconv2d_bwd_dw_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64, _i64, _int, _int, _int, _int, _int, _int,
                                                         _int]),
    "dwconv2d_bwd_dw": (_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _int, _int, _int, _int, _int, _int,
                               _int, _int, _vp, ctypes.c_size_t, _vp]),
    "dw_status_string": (ctypes.c_char_p, [_int]),
    "dw_last_cuda_error": (_int, []),
    "dw_device_error": (_int, []),
    "dw_selftest_wait_timeout": (_int, [_vp, _vp]),
}


class DwError(RuntimeError):
    """A non-OK dw_status_t from the library."""

    def __init__(self, fn, status):
        self.status = int(status)
        msg = lib().dw_status_string(self.status).decode()
        if self.status == DW_ERR_CUDA:
            msg += f" (cudaError {lib().dw_last_cuda_error()})"
        super().__init__(f"{fn}: {msg}")


def lib():
    """The loaded CUDA library (raises ImportError if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(library_path):
                raise ImportError(f"{library_path} is missing: build it with "
                                  "`python -m speech_encoder_depthwise_b200.build`")
            handle = ctypes.CDLL(library_path)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(handle, name)
                f.restype = res
                f.argtypes = args
            _lib = handle
    return _lib


def _check(fn, status):
    if status != DW_OK:
        raise DwError(fn, status)


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return DW_BF16
    if t.dtype == torch.float32:
        return DW_F32
    if t.dtype == torch.float16:
        return DW_F16
    raise TypeError(f"unsupported dtype {t.dtype}: bfloat16, float16 or float32")


def _dev(t, name, dtype=None, shape=None):
    """Device pointer of a contiguous CUDA tensor of the given dtype and shape (None: absent)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


def _stream(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def dw_status_string(status: int) -> str:
    return lib().dw_status_string(int(status)).decode()


def dw_device_error() -> int:
    """Reads and clears the kernels' device error words (synchronous); DW_OK if none was set."""
    return int(lib().dw_device_error())


def dwconv1d_fwd(x, w, bias, y, lengths, pad_left, stream=None):
    """y[b,t,c] = [t<len_b] (bias[c] + sum_k xpad[b,t+k,c] w[k,c]) into ``y``."""
    import torch
    B, T, C = x.shape
    K = w.shape[0]
    st = lib().dwconv1d_fwd(_dev(x, "x"), _dev(w, "w", torch.float32, (K, C)),
                            _dev(bias, "bias", torch.float32, (C,)), _dev(y, "y", x.dtype, x.shape),
                            _dev(lengths, "lengths", torch.int32, (B,)), B, T, C, K, int(pad_left),
                            _dtype_code(x), _stream(stream))
    _check("dwconv1d_fwd", st)


def dwconv1d_bwd(x, dy, w, dx, gw, gb, lengths, pad_left, workspace, stream=None):
    """dx and dW/dbias of dwconv1d_fwd in one pass over dy (dbias ``gb`` may be None)."""
    import torch
    B, T, C = x.shape
    K = w.shape[0]
    st = lib().dwconv1d_bwd(_dev(x, "x"), _dev(dy, "dy", x.dtype, x.shape), _dev(w, "w", torch.float32, (K, C)),
                            _dev(dx, "dx", x.dtype, x.shape), _dev(gw, "dw", torch.float32, (K, C)),
                            _dev(gb, "dbias", torch.float32, (C,)), _dev(lengths, "lengths", torch.int32, (B,)),
                            B, T, C, K, int(pad_left), _dtype_code(x), _dev(workspace, "workspace"),
                            workspace.numel() * workspace.element_size() if workspace is not None else 0,
                            _stream(stream))
    _check("dwconv1d_bwd", st)


def dwconv1d_stream_fwd(x, w, bias, y, cache, lengths, stream=None):
    """One chunk of the streaming causal conv: ``y`` from the chunk ``x`` [B,T,C] and each
    stream's K-1 cached frames; ``cache`` [B,K-1,C] is rewritten with the K-1 newest frames."""
    import torch
    B, T, C = x.shape
    K = w.shape[0]
    cache_ptr = _dev(cache, "cache", x.dtype, (B, K - 1, C)) if K > 1 else _dev(cache, "cache")
    st = lib().dwconv1d_stream_fwd(_dev(x, "x"), _dev(w, "w", torch.float32, (K, C)),
                                   _dev(bias, "bias", torch.float32, (C,)), _dev(y, "y", x.dtype, x.shape),
                                   cache_ptr, _dev(lengths, "lengths", torch.int32, (B,)), B, T, C, K,
                                   _dtype_code(x), _stream(stream))
    _check("dwconv1d_stream_fwd", st)


def dwconv1d_fwd_packed(x, w, bias, y, offsets, pad_left, stream=None):
    """Depthwise conv1d over a packed batch: x, y ``[N, C]``, sequence b on rows
    ``offsets[b]:offsets[b+1]`` (``offsets`` int32 ``[B+1]`` on the device)."""
    import torch
    N, C = x.shape
    K = w.shape[0]
    st = lib().dwconv1d_fwd_packed(_dev(x, "x"), _dev(w, "w", torch.float32, (K, C)),
                                   _dev(bias, "bias", torch.float32, (C,)), _dev(y, "y", x.dtype, (N, C)),
                                   _dev(offsets, "offsets", torch.int32), offsets.numel() - 1, N, C, K, pad_left,
                                   _dtype_code(x), _stream(stream))
    _check("dwconv1d_fwd_packed", st)


def dwconv1d_bwd_dx_packed(dy, w, dx, offsets, pad_left, stream=None):
    """Data gradient of ``dwconv1d_fwd_packed``."""
    import torch
    N, C = dy.shape
    K = w.shape[0]
    st = lib().dwconv1d_bwd_dx_packed(_dev(dy, "dy"), _dev(w, "w", torch.float32, (K, C)),
                                      _dev(dx, "dx", dy.dtype, (N, C)), _dev(offsets, "offsets", torch.int32),
                                      offsets.numel() - 1, N, C, K, pad_left, _dtype_code(dy), _stream(stream))
    _check("dwconv1d_bwd_dx_packed", st)


def dwconv1d_bwd_dw_packed_workspace_size(B, N, C, K) -> int:
    """Bytes of workspace ``dwconv1d_bwd_dw_packed`` needs."""
    return int(lib().dwconv1d_bwd_dw_packed_workspace_size(B, N, C, K))


def dwconv1d_bwd_dw_packed(x, dy, dw_, dbias, offsets, pad_left, workspace, stream=None):
    """Weight and bias gradients of ``dwconv1d_fwd_packed`` into dw_ [K, C] and dbias [C] (float32)."""
    import torch
    N, C = x.shape
    K = dw_.shape[0]
    st = lib().dwconv1d_bwd_dw_packed(_dev(x, "x"), _dev(dy, "dy", x.dtype, (N, C)),
                                      _dev(dw_, "dw", torch.float32, (K, C)), _dev(dbias, "dbias", torch.float32, (C,)),
                                      _dev(offsets, "offsets", torch.int32), offsets.numel() - 1, N, C, K, pad_left,
                                      _dtype_code(x), _dev(workspace, "workspace"),
                                      workspace.numel() * workspace.element_size() if workspace is not None else 0,
                                      _stream(stream))
    _check("dwconv1d_bwd_dw_packed", st)


def dwconv1d_bwd_dx(dy, w, dx, lengths, pad_left, stream=None):
    """Data gradient of dwconv1d_fwd into ``dx`` (pad_left is the forward pass's)."""
    import torch
    B, T, C = dy.shape
    K = w.shape[0]
    st = lib().dwconv1d_bwd_dx(_dev(dy, "dy"), _dev(w, "w", torch.float32, (K, C)),
                               _dev(dx, "dx", dy.dtype, dy.shape), _dev(lengths, "lengths", torch.int32, (B,)),
                               B, T, C, K, int(pad_left), _dtype_code(dy), _stream(stream))
    _check("dwconv1d_bwd_dx", st)


def dwconv1d_bwd_dw_workspace_size(B, T, C, K) -> int:
    return int(lib().dwconv1d_bwd_dw_workspace_size(int(B), int(T), int(C), int(K)))


def dwconv1d_bwd_dw(x, dy, dw, dbias, lengths, pad_left, workspace, stream=None):
    """Weight and bias gradients into ``dw [K, C]`` and ``dbias [C]`` (float32)."""
    import torch
    B, T, C = x.shape
    K = dw.shape[0]
    ws_ptr = _dev(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib().dwconv1d_bwd_dw(_dev(x, "x"), _dev(dy, "dy", x.dtype, x.shape),
                               _dev(dw, "dw", torch.float32, (K, C)), _dev(dbias, "dbias", torch.float32, (C,)),
                               _dev(lengths, "lengths", torch.int32, (B,)), B, T, C, K, int(pad_left),
                               _dtype_code(x), ws_ptr, ws_bytes, _stream(stream))
    _check("dwconv1d_bwd_dw", st)


def dwconv1d_bwd_dw_noalloc(x, dy, dw, dbias, lengths, pad_left, stream=None):
    """dwconv1d_bwd_dw without a workspace, for callers that cannot allocate device memory: the
    library's own 2 MiB device scratch holds the partial sums (shared by all calls; calls that
    overlap on the GPU race on it)."""
    import torch
    B, T, C = x.shape
    K = dw.shape[0]
    st = lib().dwconv1d_bwd_dw_noalloc(_dev(x, "x"), _dev(dy, "dy", x.dtype, x.shape),
                                       _dev(dw, "dw", torch.float32, (K, C)),
                                       _dev(dbias, "dbias", torch.float32, (C,)),
                                       _dev(lengths, "lengths", torch.int32, (B,)), B, T, C, K, int(pad_left),
                                       _dtype_code(x), _stream(stream))
    _check("dwconv1d_bwd_dw_noalloc", st)


def subsample_out_shape(T, F):
    """(T4, F4): two stride-2, 3-tap stages with two frames of padding each."""
    def s2(n):
        return (n - 1) // 2 + 1 if n >= 1 else 0
    return s2(s2(T)), s2(s2(F))


def dw_subsample_fwd(mel, w0, b0, w1, b1, out, lengths, out_lengths, causal, stream=None):
    """Fused conv0 + bias + ReLU + mask + depthwise conv_dw1 + bias + mask into ``out [B,T4,F4,C]``."""
    _subsample_fwd("dw_subsample_fwd", mel, w0, b0, w1, b1, out, lengths, out_lengths, causal, stream)


def dw_subsample_fwd_simt(mel, w0, b0, w1, b1, out, lengths, out_lengths, causal, stream=None):
    """``dw_subsample_fwd`` computed entirely on the FP32 FMA pipes (no tensor cores)."""
    _subsample_fwd("dw_subsample_fwd_simt", mel, w0, b0, w1, b1, out, lengths, out_lengths, causal, stream)


def _subsample_fwd(name, mel, w0, b0, w1, b1, out, lengths, out_lengths, causal, stream):
    import torch
    B, T, F = mel.shape
    C = w0.shape[-1]
    T4, F4 = subsample_out_shape(T, F)
    st = getattr(lib(), name)(
        _dev(mel, "mel", torch.float32), _dev(w0, "w0", torch.float32, (3, 3, C)),
        _dev(b0, "b0", torch.float32, (C,)), _dev(w1, "w1", torch.float32, (3, 3, C)),
        _dev(b1, "b1", torch.float32, (C,)), _dev(out, "out", None, (B, T4, F4, C)),
        _dev(lengths, "lengths", torch.int32, (B,)), _dev(out_lengths, "out_lengths", torch.int32, (B,)),
        B, T, F, C, int(bool(causal)), _dtype_code(out), _stream(stream))
    _check(name, st)


def dw_subsample_bwd_workspace_size(B, T, F, C):
    """Bytes of workspace ``dw_subsample_bwd`` needs for these sizes."""
    return int(lib().dw_subsample_bwd_workspace_size(B, T, F, C))


def dw_subsample_bwd(mel, w0, b0, w1, dout, lengths, dw0, db0, dw1, db1, causal, workspace, stream=None):
    """Gradients of sum(out * dout) of the fused subsampler into dw0/db0/dw1/db1 (float32)."""
    import torch
    B, T, F = mel.shape
    C = w0.shape[-1]
    T4, F4 = subsample_out_shape(T, F)
    st = lib().dw_subsample_bwd(_dev(mel, "mel", torch.float32), _dev(w0, "w0", torch.float32, (3, 3, C)),
                                _dev(b0, "b0", torch.float32, (C,)), _dev(w1, "w1", torch.float32, (3, 3, C)),
                                _dev(dout, "dout", None, (B, T4, F4, C)), _dev(lengths, "lengths", torch.int32, (B,)),
                                _dev(dw0, "dw0", torch.float32, (3, 3, C)), _dev(db0, "db0", torch.float32, (C,)),
                                _dev(dw1, "dw1", torch.float32, (3, 3, C)), _dev(db1, "db1", torch.float32, (C,)),
                                B, T, F, C, int(bool(causal)), _dtype_code(dout), _dev(workspace, "workspace"),
                                workspace.numel() * workspace.element_size() if workspace is not None else 0,
                                _stream(stream))
    _check("dw_subsample_bwd", st)


def conv2d_out_shape(T, F, KT, KF, stride, pads):
    """(To, Fo) of ``dwconv2d_fwd``: (n + pads - k) // s + 1 per axis, 0 when the window does not fit."""
    (st, sf), (pt, pb, pf) = stride, pads

    def o(n, p0, p1, k, s):
        m = n + p0 + p1 - k
        return 0 if m < 0 else m // s + 1
    return o(T, pt, pb, KT, st), o(F, pf, pf, KF, sf)


def _c2_geom(stride, pads):
    (st, sf), (pt, pb, pf) = stride, pads
    return int(st), int(sf), int(pt), int(pb), int(pf)


def dwconv2d_fwd(x, w, bias, y, lengths, out_lengths, stride, pads, stream=None):
    """Depthwise conv2d of channels-last x [B,T,F,C] with taps w [KT,KF,C] (float32) into
    y [B,To,Fo,C]; ``stride`` = (st, sf), ``pads`` = (pad_t, pad_b, pad_f)."""
    import torch
    B, T, F, C = x.shape
    KT, KF = w.shape[:2]
    To, Fo = conv2d_out_shape(T, F, KT, KF, stride, pads)
    st = lib().dwconv2d_fwd(_dev(x, "x"), _dev(w, "w", torch.float32, (KT, KF, C)),
                            _dev(bias, "bias", torch.float32, (C,)), _dev(y, "y", x.dtype, (B, To, Fo, C)),
                            _dev(lengths, "lengths", torch.int32, (B,)),
                            _dev(out_lengths, "out_lengths", torch.int32, (B,)), B, T, F, C, KT, KF,
                            *_c2_geom(stride, pads), _dtype_code(x), _stream(stream))
    _check("dwconv2d_fwd", st)


def dwconv2d_bwd_dx(dy, w, dx, lengths, stride, pads, stream=None):
    """Data gradient of ``dwconv2d_fwd`` into dx [B,T,F,C] from dy [B,To,Fo,C]."""
    import torch
    B, T, F, C = dx.shape
    KT, KF = w.shape[:2]
    To, Fo = conv2d_out_shape(T, F, KT, KF, stride, pads)
    st = lib().dwconv2d_bwd_dx(_dev(dy, "dy", dx.dtype, (B, To, Fo, C)), _dev(w, "w", torch.float32, (KT, KF, C)),
                               _dev(dx, "dx"), _dev(lengths, "lengths", torch.int32, (B,)), B, T, F, C, KT, KF,
                               *_c2_geom(stride, pads), _dtype_code(dx), _stream(stream))
    _check("dwconv2d_bwd_dx", st)


def dwconv2d_bwd_dw_workspace_size(B, T, F, C, KT, KF, stride, pads) -> int:
    """Bytes of workspace ``dwconv2d_bwd_dw`` needs for these sizes."""
    return int(lib().dwconv2d_bwd_dw_workspace_size(B, T, F, C, KT, KF, *_c2_geom(stride, pads)))


def dwconv2d_bwd_dw(x, dy, dw, dbias, lengths, stride, pads, workspace, stream=None):
    """Weight and bias gradients of ``dwconv2d_fwd`` into dw [KT,KF,C] and dbias [C] (float32)."""
    import torch
    B, T, F, C = x.shape
    KT, KF = dw.shape[:2]
    To, Fo = conv2d_out_shape(T, F, KT, KF, stride, pads)
    st = lib().dwconv2d_bwd_dw(_dev(x, "x"), _dev(dy, "dy", x.dtype, (B, To, Fo, C)),
                               _dev(dw, "dw", torch.float32, (KT, KF, C)), _dev(dbias, "dbias", torch.float32, (C,)),
                               _dev(lengths, "lengths", torch.int32, (B,)), B, T, F, C, KT, KF,
                               *_c2_geom(stride, pads), _dtype_code(x), _dev(workspace, "workspace"),
                               workspace.numel() * workspace.element_size() if workspace is not None else 0,
                               _stream(stream))
    _check("dwconv2d_bwd_dw", st)


def dw_selftest_wait_timeout(done, stream=None):
    """Launch the bounded-wait self-test: ``done`` (int32 CUDA tensor of 1) receives 2 once the
    wait has given up; ``dw_device_error()`` then returns DW_ERR_TIMEOUT (and clears it)."""
    import torch
    _check("dw_selftest_wait_timeout", lib().dw_selftest_wait_timeout(_dev(done, "done", torch.int32, (1,)),
                                                                      _stream(stream)))
