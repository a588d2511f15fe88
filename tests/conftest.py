import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running test")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.fixture(autouse=True, scope="session")
def _short_device_waits():
    """Device-side waits in tests give up after 1 s instead of the default 2 s."""
    try:
        import torch
        if torch.cuda.is_available():
            import exact_io_aware_44_b200 as fa
            fa.set_wait_budget_ns(1_000_000_000)
    except ImportError:
        pass
    yield
