import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def _gpu_selected(config):
    """True when the run selected the GPU tests on purpose (-m gpu)."""
    expr = (config.getoption("markexpr", default="") or "").replace(" ", "")
    return "gpu" in expr and "notgpu" not in expr


@pytest.fixture(scope="session")
def cuda_ok(request):
    """GPU tests need a CUDA device.  Without one they are skipped in a general run,
    but fail when they were selected with -m gpu: such a run would otherwise pass
    without testing anything."""
    import torch
    if not torch.cuda.is_available():
        if _gpu_selected(request.config):
            pytest.fail("-m gpu selected but no CUDA device is available")
        pytest.skip("no CUDA device")
    return True
