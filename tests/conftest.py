import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA GPU (B200, sm_100a); runs the CUDA path through the C ABI")


@pytest.fixture(scope="session", autouse=True)
def _oracle_built():
    import oracle
    oracle.build()


@pytest.fixture(scope="session")
def ssm():
    """The CUDA binding, failing loudly when no GPU or no library is present."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("gpu test run without a visible CUDA device")
    from selective_state_space_25_b200 import ssmscan
    return ssmscan


@pytest.fixture(autouse=True)
def _debug_bounds_word(request):
    """With SSM_DEBUG_BOUNDS=1 (the debug-bounds library) every GPU test ends
    by reading the device's bounds word, so a miss is reported by the test
    whose kernels made it."""
    yield
    if os.environ.get("SSM_DEBUG_BOUNDS") == "1" and request.node.get_closest_marker("gpu"):
        from selective_state_space_25_b200 import ssmscan
        ssmscan.check_device_errors()
