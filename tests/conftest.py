import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test collected without a CUDA device")
    return torch.device("cuda:0")


@pytest.fixture(autouse=True)
def _no_failed_bounds_check(request):
    """With ZB_DEBUG=1 the GPU tests run on the bounds-checked library; each
    must leave its record of failed checks empty (a test that provokes one
    reads and clears the record itself)."""
    yield
    if os.environ.get("ZB_DEBUG") != "1" or request.node.get_closest_marker("gpu") is None:
        return
    from token_dispatch_top_b200 import zb
    if zb._lib is None:
        return
    rec = zb.debug_read(reset=True)
    assert rec["count"] == 0, f"failed bounds checks: {rec}"
