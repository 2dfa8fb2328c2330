"""Every entry point can be captured into a CUDA graph (no synchronization, no allocation, no
host read-back inside a call) and the replayed graph produces exactly the eager results.
The workspace-free dW is called once before capture, as its documentation asks."""
import numpy as np
import pytest
import torch

import speech_encoder_depthwise_b200 as dw
from gpuhelp import dev
from synth import conv1d_inputs, conv2d_inputs, subsample_inputs

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from speech_encoder_depthwise_b200 import build
    build.build()
    dw.lib()


def test_every_entry_point_replays_exactly():
    B, T, C, K, pl = 4, 300, 256, 9, 4
    d = conv1d_inputs(B, T, C, K, dtype="bf16", len_range=(100, 300), seed=3, with_dy=True)
    x, g, w, b, ln = dev(d["x"], BF), dev(d["dy"], BF), dev(d["w"]), dev(d["bias"]), dev(d["lengths"])
    s = subsample_inputs(2, 64, 80, 256, len_range=(30, 64), seed=4)
    mel, w0, b0, w1, b1, sl = (dev(s["mel"]), dev(s["w0"]), dev(s["b0"]), dev(s["w1"]), dev(s["b1"]),
                               dev(s["lengths"]))
    T4, F4 = dw.subsample_out_shape(64, 80)
    dout = torch.randn(2, T4, F4, 256, device="cuda").to(BF)
    To, Fo = dw.conv2d_out_shape(40, 20, 3, 3, (2, 2), (1, 1, 1))
    c2 = conv2d_inputs(2, 40, 20, 128, 3, 3, dtype="bf16", len_range=(20, 40), seed=5, dy_shape=(2, To, Fo, 128))
    x2, g2, wc, bc, l2 = (dev(c2["x"], BF), dev(c2["dy"], BF), dev(c2["w"]), dev(c2["bias"]), dev(c2["lengths"]))
    lens = np.clip(d["lengths"], 0, T)
    xp = torch.cat([x[i, :int(lens[i])] for i in range(B)])
    off = dev(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32))

    def outputs():
        return dict(y=torch.empty_like(x), dx=torch.empty_like(x), dx2=torch.empty_like(x),
                    gw=torch.empty(K, C, device="cuda"), gb=torch.empty(C, device="cuda"),
                    gw2=torch.empty(K, C, device="cuda"), gb2=torch.empty(C, device="cuda"),
                    gw3=torch.empty(K, C, device="cuda"), gb3=torch.empty(C, device="cuda"),
                    cache=torch.zeros(B, K - 1, C, dtype=BF, device="cuda"), ys=torch.empty(B, 8, C, dtype=BF, device="cuda"),
                    out=torch.empty(2, T4, F4, 256, dtype=BF, device="cuda"), ol=torch.empty(2, dtype=torch.int32, device="cuda"),
                    sg=[torch.empty(3, 3, 256, device="cuda"), torch.empty(256, device="cuda"),
                        torch.empty(3, 3, 256, device="cuda"), torch.empty(256, device="cuda")],
                    y2=torch.empty(2, To, Fo, 128, dtype=BF, device="cuda"), dx2d=torch.empty_like(x2),
                    gw2d=torch.empty(3, 3, 128, device="cuda"), gb2d=torch.empty(128, device="cuda"),
                    yp=torch.empty_like(xp), gwp=torch.empty(K, C, device="cuda"), gbp=torch.empty(C, device="cuda"))

    ws = torch.empty(dw.dwconv1d_bwd_dw_workspace_size(B, T, C, K), dtype=torch.uint8, device="cuda")
    ws_s = torch.empty(dw.dw_subsample_bwd_workspace_size(2, 64, 80, 256), dtype=torch.uint8, device="cuda")
    ws_2 = torch.empty(dw.dwconv2d_bwd_dw_workspace_size(2, 40, 20, 128, 3, 3, (2, 2), (1, 1, 1)), dtype=torch.uint8,
                       device="cuda")
    ws_p = torch.empty(dw.dwconv1d_bwd_dw_packed_workspace_size(B, xp.shape[0], C, K), dtype=torch.uint8, device="cuda")

    def run(o):
        dw.dwconv1d_fwd(x, w, b, o["y"], ln, pl)
        dw.dwconv1d_bwd_dx(g, w, o["dx"], ln, pl)
        dw.dwconv1d_bwd_dw(x, g, o["gw"], o["gb"], ln, pl, ws)
        dw.dwconv1d_bwd(x, g, w, o["dx2"], o["gw2"], o["gb2"], ln, pl, ws)
        dw.dwconv1d_bwd_dw_noalloc(x, g, o["gw3"], o["gb3"], ln, pl)
        dw.dwconv1d_stream_fwd(x[:, :8].contiguous(), w, b, o["ys"], o["cache"], None)
        dw.dw_subsample_fwd(mel, w0, b0, w1, b1, o["out"], sl, o["ol"], 0)
        dw.dw_subsample_bwd(mel, w0, b0, w1, dout, sl, *o["sg"], 0, ws_s)
        dw.dwconv2d_fwd(x2, wc, bc, o["y2"], l2, None, (2, 2), (1, 1, 1))
        dw.dwconv2d_bwd_dx(g2, wc, o["dx2d"], l2, (2, 2), (1, 1, 1))
        dw.dwconv2d_bwd_dw(x2, g2, o["gw2d"], o["gb2d"], l2, (2, 2), (1, 1, 1), ws_2)
        dw.dwconv1d_fwd_packed(xp, w, b, o["yp"], off, pl)
        dw.dwconv1d_bwd_dw_packed(xp, xp, o["gwp"], o["gbp"], off, pl, ws_p)

    eager = outputs()
    run(eager)  # also the workspace-free dW's first call, before any capture
    torch.cuda.synchronize()
    replayed = outputs()
    s_cap = torch.cuda.Stream()
    with torch.cuda.stream(s_cap):
        graph = torch.cuda.CUDAGraph()
        graph.capture_begin()
        run(replayed)
        graph.capture_end()
        graph.replay()
    torch.cuda.synchronize()
    for k in eager:
        a, r = eager[k], replayed[k]
        for u, v in (zip(a, r) if isinstance(a, list) else [(a, r)]):
            assert torch.equal(u, v), f"{k} differs between eager and graph replay"
    assert dw.dw_device_error() == dw.DW_OK
