import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_device():
    """The first CUDA device; skips on a host without one."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device on this host")
    return torch.device("cuda:0")


@pytest.fixture(autouse=True)
def _no_device_error(request):
    """After every GPU test: no kernel recorded a timed-out wait."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    import speech_encoder_depthwise_b200 as dw
    assert dw.dw_device_error() == dw.DW_OK, "a kernel's bounded wait gave up (DW_ERR_TIMEOUT)"
