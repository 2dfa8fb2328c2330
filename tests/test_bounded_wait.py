"""The bounded waits give up instead of hanging: a one-block kernel waits on an mbarrier that
nothing completes; its wait runs out after the poll limit, the kernel records the error and
returns, dw_device_error() reports DW_ERR_TIMEOUT once (then DW_OK), and the context keeps
working (a forward conv afterwards still matches the oracle).  No fault is raised."""
import time

import numpy as np
import pytest
import torch

import oracle
import speech_encoder_depthwise_b200 as dw
from gpuhelp import assert_bf16_close, dev
from synth import conv1d_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from speech_encoder_depthwise_b200 import build
    build.build()
    dw.lib()


def test_wait_gives_up_and_reports_timeout():
    done = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    dw.dw_selftest_wait_timeout(done)
    torch.cuda.synchronize()
    waited = time.time() - t0
    assert int(done.item()) == 2, "the wait should have given up"
    assert dw.dw_device_error() == dw.DW_ERR_TIMEOUT
    assert dw.dw_device_error() == dw.DW_OK          # read and cleared
    assert waited < 60.0
    d = conv1d_inputs(2, 100, 64, 9, dtype="bf16", len_range=(50, 100), seed=1)
    y = torch.empty(2, 100, 64, dtype=torch.bfloat16, device="cuda")
    dw.dwconv1d_fwd(dev(d["x"], torch.bfloat16), dev(d["w"]), dev(d["bias"]), y, dev(d["lengths"]), 4)
    torch.cuda.synchronize()
    assert_bf16_close(y.float().cpu().numpy(), oracle.dwconv1d_fwd(d["x"], d["w"], d["bias"], d["lengths"], 4))
