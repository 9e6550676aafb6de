import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload checks")


@pytest.fixture(scope="session")
def cuda_device():
    import torch

    assert torch.cuda.is_available(), "GPU test collected on a machine without CUDA"
    major, minor = torch.cuda.get_device_capability(0)
    assert (major, minor) == (10, 0), f"needs sm_100 (B200), got sm_{major}{minor}"
    return torch.device("cuda", 0)
