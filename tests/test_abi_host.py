"""Host-side checks of the C ABI, runnable without a GPU.

The library is built here (nvcc cross-compiles for sm_100a), loaded, and checked to export
every function that include/dwconv.h declares.  Invalid arguments are rejected on the host
before any CUDA call, so those paths run on a machine with no device.  Pointers in these
calls are fake addresses that the library compares but never dereferences.
"""
import ctypes
import os
import re

import pytest

import speech_encoder_depthwise_b200 as dw
from speech_encoder_depthwise_b200 import build as dwbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "dwconv.h")


@pytest.fixture(scope="module")
def lib():
    dwbuild.build()
    return dw.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "defined")))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("dwconv1d_fwd", "dwconv1d_bwd_dx", "dwconv1d_bwd_dw_workspace_size", "dwconv1d_bwd_dw",
              "dw_subsample_fwd", "dw_status_string", "dw_last_cuda_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in dwconv.h but not exported"
        assert n in dw.SIGNATURES, f"{n} has no binding signature"


def test_status_strings(lib):
    for code in range(6):
        assert dw.dw_status_string(code).startswith("DW_")
    assert "unknown" in dw.dw_status_string(99)


FAKE_X, FAKE_W, FAKE_Y, FAKE_WS = 0x10000000, 0x20000000, 0x30000000, 0x40000000


def fwd(lib, x=FAKE_X, w=FAKE_W, b=None, y=FAKE_Y, ln=None, B=2, T=10, C=8, K=3, pl=1, dt=dw.DW_BF16):
    return lib.dwconv1d_fwd(x, w, b, y, ln, B, T, C, K, pl, dt, None)


@pytest.mark.parametrize("kw", [dict(x=None), dict(w=None), dict(y=None), dict(K=0), dict(K=-3),
                                dict(pl=-1), dict(pl=3), dict(B=-1), dict(T=-1), dict(C=0),
                                dict(dt=7), dict(y=FAKE_X), dict(y=FAKE_X + 20),
                                dict(B=1 << 40, T=1 << 40)])
def test_fwd_rejects_invalid_arguments(lib, kw):
    assert fwd(lib, **kw) == dw.DW_ERR_INVALID_ARG


def test_dx_rejects_invalid_arguments(lib):
    f = lib.dwconv1d_bwd_dx
    assert f(None, FAKE_W, FAKE_Y, None, 2, 10, 8, 3, 1, dw.DW_BF16, None) == dw.DW_ERR_INVALID_ARG
    assert f(FAKE_X, FAKE_W, FAKE_X, None, 2, 10, 8, 3, 1, dw.DW_BF16, None) == dw.DW_ERR_INVALID_ARG
    assert f(FAKE_X, FAKE_W, FAKE_Y, None, 2, 10, 8, 3, 5, dw.DW_F32, None) == dw.DW_ERR_INVALID_ARG


def test_stream_rejects_invalid_arguments(lib):
    f = lib.dwconv1d_stream_fwd
    FAKE_C = 0x50000000
    ok = (FAKE_X, FAKE_W, None, FAKE_Y, FAKE_C, None, 4, 16, 512, 9, dw.DW_BF16, None)

    def call(**kw):
        a = list(ok)
        for k, v in kw.items():
            a[["x", "w", "bias", "y", "cache", "ln", "B", "T", "C", "K", "dt", "s"].index(k)] = v
        return f(*a)
    assert call(cache=None) == dw.DW_ERR_INVALID_ARG             # K > 1 needs a cache
    assert call(cache=FAKE_Y + 64) == dw.DW_ERR_INVALID_ARG      # cache overlaps y
    assert call(cache=FAKE_X) == dw.DW_ERR_INVALID_ARG           # cache overlaps x
    assert call(y=FAKE_X + 2) == dw.DW_ERR_INVALID_ARG           # y overlaps x
    assert call(K=0) == dw.DW_ERR_INVALID_ARG
    assert call(C=0) == dw.DW_ERR_INVALID_ARG
    assert call(B=-1) == dw.DW_ERR_INVALID_ARG
    assert call(dt=3) == dw.DW_ERR_INVALID_ARG
    assert call(K=5000) == dw.DW_ERR_UNSUPPORTED
    assert call(T=0, x=None, y=None) == dw.DW_OK                 # no frames: nothing to do
    assert call(B=0) == dw.DW_OK


def test_fp16_is_accepted_and_unknown_dtypes_are_not(lib):
    assert fwd(lib, B=0, dt=dw.DW_F16) == dw.DW_OK
    assert fwd(lib, x=None, dt=dw.DW_F16) == dw.DW_ERR_INVALID_ARG
    assert fwd(lib, dt=3) == dw.DW_ERR_INVALID_ARG
    assert lib.dwconv2d_fwd(FAKE_X, FAKE_W, None, FAKE_Y, None, None, 0, 40, 20, 8, 3, 3, 2, 2, 1, 1, 1,
                            dw.DW_F16, None) == dw.DW_OK


def test_packed_rejects_invalid_arguments(lib):
    f = lib.dwconv1d_fwd_packed
    OFF = 0x60000000
    ok = [FAKE_X, FAKE_W, None, FAKE_Y, OFF, 4, 100, 64, 9, 4, dw.DW_BF16, None]
    names = ["x", "w", "bias", "y", "off", "B", "N", "C", "K", "pl", "dt", "s"]

    def call(fn=f, **kw):
        a = list(ok)
        for k, v in kw.items():
            a[names.index(k)] = v
        return fn(*a)
    assert call(off=None) == dw.DW_ERR_INVALID_ARG
    assert call(x=None) == dw.DW_ERR_INVALID_ARG
    assert call(y=FAKE_X + 16) == dw.DW_ERR_INVALID_ARG      # y overlaps x
    assert call(B=-1) == dw.DW_ERR_INVALID_ARG
    assert call(pl=9) == dw.DW_ERR_INVALID_ARG
    assert call(dt=7) == dw.DW_ERR_INVALID_ARG
    assert call(N=1 << 30, y=1 << 44) == dw.DW_ERR_UNSUPPORTED
    assert call(B=0, off=None) == dw.DW_OK
    assert call(N=0, x=None, y=None) == dw.DW_OK
    n = lib.dwconv1d_bwd_dw_packed_workspace_size(4, 100, 64, 9)
    assert n > 0 and n % 16 == 0 and lib.dwconv1d_bwd_dw_packed_workspace_size(4, 100, 0, 9) == 0
    h = lib.dwconv1d_bwd_dw_packed
    args = (FAKE_X, FAKE_Y, FAKE_W, None, OFF, 4, 100, 64, 9, 4, dw.DW_BF16)
    assert h(*args, None, n, None) == dw.DW_ERR_WORKSPACE
    assert h(*args, FAKE_WS, n - 16, None) == dw.DW_ERR_WORKSPACE
    assert h(*args, FAKE_W, n, None) == dw.DW_ERR_INVALID_ARG           # workspace overlaps dW
    assert h(FAKE_X, FAKE_Y, FAKE_W, None, None, 4, 100, 64, 9, 4, dw.DW_BF16, FAKE_WS, n, None) \
        == dw.DW_ERR_INVALID_ARG                                         # no offsets
    assert h(FAKE_X, FAKE_Y, None, None, OFF, 4, 100, 64, 9, 4, dw.DW_BF16, FAKE_WS, n, None) \
        == dw.DW_ERR_INVALID_ARG
    g = lib.dwconv1d_bwd_dx_packed
    assert g(FAKE_X, FAKE_W, FAKE_Y, None, 4, 100, 64, 9, 4, dw.DW_BF16, None) == dw.DW_ERR_INVALID_ARG
    assert g(FAKE_X, FAKE_W, FAKE_X, OFF, 4, 100, 64, 9, 4, dw.DW_BF16, None) == dw.DW_ERR_INVALID_ARG


def test_empty_inputs_are_noops_without_a_device(lib):
    assert fwd(lib, B=0) == dw.DW_OK
    assert fwd(lib, T=0) == dw.DW_OK
    assert fwd(lib, x=None, y=None, B=0) == dw.DW_OK
    assert lib.dwconv1d_bwd_dx(None, None, None, None, 3, 0, 8, 9, 4, dw.DW_BF16, None) == dw.DW_OK


def test_dw_workspace_rules(lib):
    n = dw.dwconv1d_bwd_dw_workspace_size(16, 1500, 512, 9)
    assert n > 0 and n % 16 == 0
    # independent of dtype and pointers, grows with K and C, zero for empty inputs
    assert dw.dwconv1d_bwd_dw_workspace_size(16, 1500, 512, 15) > n
    assert dw.dwconv1d_bwd_dw_workspace_size(0, 1500, 512, 9) == 0
    assert dw.dwconv1d_bwd_dw_workspace_size(16, 0, 512, 9) == 0
    f = lib.dwconv1d_bwd_dw
    args = (FAKE_X, FAKE_Y, FAKE_W, None, None, 16, 1500, 512, 9, 4, dw.DW_BF16)
    assert f(*args, None, n, None) == dw.DW_ERR_WORKSPACE
    assert f(*args, FAKE_WS, n - 4, None) == dw.DW_ERR_WORKSPACE
    assert f(*args, FAKE_WS + 4, n, None) == dw.DW_ERR_WORKSPACE
    # workspace overlapping the output
    assert f(*args, FAKE_W, n, None) == dw.DW_ERR_INVALID_ARG
    assert f(FAKE_X, FAKE_Y, None, None, None, 16, 1500, 512, 9, 4, dw.DW_BF16, FAKE_WS, n, None) \
        == dw.DW_ERR_INVALID_ARG
    assert f(*args[:9], 9, dw.DW_BF16, FAKE_WS, n, None) == dw.DW_ERR_INVALID_ARG


@pytest.mark.parametrize("entry", ["dw_subsample_fwd", "dw_subsample_fwd_simt"])
def test_subsample_rejects_invalid_arguments(lib, entry):
    f = getattr(lib, entry)
    ok = [FAKE_X, FAKE_W, FAKE_W + 4096, FAKE_W + 8192, FAKE_W + 12288, FAKE_Y, None, None,
          2, 40, 16, 8, 0, dw.DW_BF16, None]

    def call(**kw):
        a = list(ok)
        for k, v in kw.items():
            a[{"mel": 0, "w0": 1, "out": 5, "B": 8, "T": 9, "F": 10, "C": 11, "causal": 12, "dt": 13}[k]] = v
        return f(*a)

    assert call(mel=None) == dw.DW_ERR_INVALID_ARG
    assert call(w0=None) == dw.DW_ERR_INVALID_ARG
    assert call(out=None) == dw.DW_ERR_INVALID_ARG
    assert call(F=0) == dw.DW_ERR_INVALID_ARG
    assert call(C=0) == dw.DW_ERR_INVALID_ARG
    assert call(B=-2) == dw.DW_ERR_INVALID_ARG
    assert call(causal=2) == dw.DW_ERR_INVALID_ARG
    assert call(dt=5) == dw.DW_ERR_INVALID_ARG
    assert call(dt=3) == dw.DW_ERR_INVALID_ARG
    assert call(out=FAKE_X) == dw.DW_ERR_INVALID_ARG       # output overlaps the mel input
    assert call(B=0) == dw.DW_OK
    assert call(T=0) == dw.DW_OK


def test_conv2d_rejects_invalid_arguments(lib):
    f = lib.dwconv2d_fwd
    names = ["x", "w", "bias", "y", "ln", "oln", "B", "T", "F", "C", "KT", "KF", "st", "sf", "pt", "pb", "pf",
             "dt", "s"]
    ok = [FAKE_X, FAKE_W, None, FAKE_Y, None, None, 2, 40, 20, 8, 3, 3, 2, 2, 1, 1, 1, dw.DW_BF16, None]

    def call(fn=f, base=ok, keys=names, **kw):
        a = list(base)
        for k, v in kw.items():
            a[keys.index(k)] = v
        return fn(*a)

    for kw in (dict(x=None), dict(w=None), dict(y=None), dict(KT=0), dict(KF=-1), dict(st=0), dict(sf=-2),
               dict(pt=-1), dict(pb=-1), dict(pf=-1), dict(B=-1), dict(T=-1), dict(F=0), dict(C=0), dict(dt=4),
               dict(y=FAKE_X + 64), dict(T=1 << 31), dict(pt=1 << 30)):
        assert call(**kw) == dw.DW_ERR_INVALID_ARG, kw
    assert call(C=1 << 23) == dw.DW_ERR_UNSUPPORTED
    assert call(B=0) == dw.DW_OK                                  # nothing to do
    assert call(T=0, x=None, y=None) == dw.DW_OK                  # no output rows, no lengths asked
    assert call(KF=30, x=None, y=None) == dw.DW_OK                # the window does not fit F
    # data gradient: dy and dx must not overlap; an empty input is a no-op
    g = lib.dwconv2d_bwd_dx
    gn = ["dy", "w", "dx", "ln", "B", "T", "F", "C", "KT", "KF", "st", "sf", "pt", "pb", "pf", "dt", "s"]
    gok = [FAKE_Y, FAKE_W, FAKE_X, None, 2, 40, 20, 8, 3, 3, 2, 2, 1, 1, 1, dw.DW_BF16, None]
    assert call(g, gok, gn, dy=None) == dw.DW_ERR_INVALID_ARG
    assert call(g, gok, gn, dx=None) == dw.DW_ERR_INVALID_ARG
    assert call(g, gok, gn, w=None) == dw.DW_ERR_INVALID_ARG
    assert call(g, gok, gn, dx=FAKE_Y + 32) == dw.DW_ERR_INVALID_ARG
    assert call(g, gok, gn, st=0) == dw.DW_ERR_INVALID_ARG
    assert call(g, gok, gn, B=0, dy=None, dx=None) == dw.DW_OK
    assert call(g, gok, gn, T=0, dy=None, dx=None) == dw.DW_OK


def test_conv2d_dw_workspace_rules(lib):
    geom = (2, 2, 1, 1, 1)
    n = lib.dwconv2d_bwd_dw_workspace_size(16, 750, 20, 256, 3, 3, *geom)
    assert n > 0 and n % 16 == 0
    assert lib.dwconv2d_bwd_dw_workspace_size(16, 750, 20, 256, 5, 5, *geom) > n
    assert lib.dwconv2d_bwd_dw_workspace_size(16, 750, 20, 512, 3, 3, *geom) > n
    assert lib.dwconv2d_bwd_dw_workspace_size(16, 750, 0, 256, 3, 3, *geom) == 0      # invalid F
    assert lib.dwconv2d_bwd_dw_workspace_size(16, 750, 20, 256, 3, 3, 0, 2, 1, 1, 1) == 0
    f = lib.dwconv2d_bwd_dw
    head = (FAKE_X, FAKE_Y, FAKE_W, None, None, 16, 750, 20, 256, 3, 3, *geom, dw.DW_BF16)
    assert f(*head, None, n, None) == dw.DW_ERR_WORKSPACE
    assert f(*head, FAKE_WS, n - 16, None) == dw.DW_ERR_WORKSPACE
    assert f(*head, FAKE_WS + 8, n, None) == dw.DW_ERR_WORKSPACE
    assert f(*head, FAKE_W - 64, n, None) == dw.DW_ERR_INVALID_ARG             # workspace overlaps dW
    assert f(FAKE_X, FAKE_Y, None, None, None, 16, 750, 20, 256, 3, 3, *geom, dw.DW_BF16, FAKE_WS, n, None) \
        == dw.DW_ERR_INVALID_ARG
    assert f(FAKE_X, FAKE_Y, FAKE_W, FAKE_W + 64, None, 16, 750, 20, 256, 3, 3, *geom, dw.DW_BF16, FAKE_WS, n,
             None) == dw.DW_ERR_INVALID_ARG                                   # dbias overlaps dW
    assert f(None, FAKE_Y, FAKE_W, None, None, 16, 750, 20, 256, 3, 3, *geom, dw.DW_BF16, FAKE_WS, n, None) \
        == dw.DW_ERR_INVALID_ARG


def test_binding_rejects_host_tensors(lib):
    import torch
    x = torch.zeros(1, 4, 2, dtype=torch.bfloat16)
    w = torch.zeros(3, 2)
    with pytest.raises(ValueError):
        dw.dwconv1d_fwd(x, w, None, x.clone(), None, 1)


def test_product_path_imports_no_oracle():
    """The CUDA library's binding never reaches the CPU oracle."""
    pkg = os.path.dirname(dw.__file__)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(root, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
