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
