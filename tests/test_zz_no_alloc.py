"""The allocation-free weight-gradient entry point, dwconv1d_bwd_dw_noalloc.

Some callers cannot allocate device memory: code embedded in a host that owns all device
memory through its own allocator and hands plug-ins no allocation handle, and streaming loops
that must not call cudaMalloc after start-up because an allocation can block on the whole
device.  For them the library keeps a 2 MiB scratch array of its own in device memory.  This
test calls that entry point through the C ABI, twice in a row, and checks each result against
the fp64 CPU oracle with the bar the other dW tests use (<= 2e-2 absolute and <= 1e-5 * RMS),
and against the workspace entry point's (dwconv1d_bwd_dw) result within float32 summation-order
rounding.  Two of the sizes hold (K+1)*C so large that the scratch takes fewer partial rows than
the workspace path would use (6 rows on 16-byte aligned rows, and a single row on the register
kernel and on the pipelined kernel), which changes the grid and the order of the sums.  The file
is collected last, and passes alone in a fresh process or after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import speech_encoder_depthwise_b200 as dw
from gpuhelp import dev, max_abs, rms
from synth import conv1d_inputs

pytestmark = pytest.mark.gpu

SCRATCH = 2 << 20


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


@pytest.fixture(scope="module")
def lib(cuda_device):
    from speech_encoder_depthwise_b200 import build
    build.build()
    return dw.lib()


CASES = [
    (16, 1500, 512, 9, 4, 1),      # the conformer workload: the scratch holds every partial row
    (3, 77, 130, 15, 14, 5),       # odd channels, causal K = 15
    (8, 1000, 8192, 9, 4, 6),      # 6 partial rows fit (the workspace path would use 32)
    (2, 400, 52424, 9, 4, 7),      # 1 row fits; rows are 16-byte aligned (pipelined kernel)
    (2, 400, 52428, 9, 4, 8),      # 1 row fits; C % 8 != 0 (register-tiled kernel)
]


@pytest.mark.parametrize("B,T,C,K,pl,seed", CASES)
def test_noalloc_matches_oracle_and_workspace_entry_point(lib, B, T, C, K, pl, seed):
    rows_fit = SCRATCH // ((K + 1) * C * 4)
    d = conv1d_inputs(B, T, C, K, dtype="bf16", len_range=(T // 2, T), seed=seed, with_dy=True)
    rdw, rdb = oracle.dwconv1d_bwd_dw(d["x"], d["dy"], K, d["lengths"], pl)
    x, g = dev(d["x"], torch.bfloat16), dev(d["dy"], torch.bfloat16)
    ln = dev(d["lengths"])
    ws_w = torch.empty(K, C, device="cuda")
    ws_b = torch.empty(C, device="cuda")
    ws = torch.empty(max(16, dw.dwconv1d_bwd_dw_workspace_size(B, T, C, K)), dtype=torch.uint8, device="cuda")
    dw.dwconv1d_bwd_dw(x, g, ws_w, ws_b, ln, pl, ws)
    torch.cuda.synchronize()
    sw, sb = ws_w.cpu().numpy().astype(np.float64), ws_b.cpu().numpy().astype(np.float64)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        gw = torch.full((K, C), float("nan"), device="cuda")
        gb = torch.full((C,), float("nan"), device="cuda")
        st = lib.dwconv1d_bwd_dw_noalloc(_ptr(x), _ptr(g), _ptr(gw), _ptr(gb), _ptr(ln), B, T, C, K, pl,
                                         dw.DW_BF16, stream)
        assert st == dw.DW_OK, dw.dw_status_string(st)
        torch.cuda.synchronize()
        for got, ref, other in ((gw.cpu().numpy(), rdw, sw), (gb.cpu().numpy(), rdb, sb)):
            e = max_abs(got, ref)
            assert e <= 2e-2 and e <= 1e-5 * max(rms(ref), 1e-6), (e, rms(ref), rows_fit)
            # the workspace path: the same sums in another order (float32 rounding apart)
            assert max_abs(got, other) <= 2e-5 * max(rms(ref), 1e-6), (max_abs(got, other), rows_fit)


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    # (K+1) * C * 4 bytes above 2 MiB: rejected on the host, pointers never touched
    fake = ctypes.c_void_p(0x10000000)
    st = lib.dwconv1d_bwd_dw_noalloc(fake, ctypes.c_void_p(0x20000000), ctypes.c_void_p(0x30000000), None, None,
                                     2, 100, 65536, 9, 4, dw.DW_BF16, None)
    assert st == dw.DW_ERR_UNSUPPORTED
    st = lib.dwconv1d_bwd_dw_noalloc(fake, ctypes.c_void_p(0x20000000), ctypes.c_void_p(0x30000000), None, None,
                                     2, 100, 52429, 9, 4, dw.DW_BF16, None)
    assert st == dw.DW_ERR_UNSUPPORTED
