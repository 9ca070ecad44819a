import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload (seconds to minutes)")

import pytest  # noqa: E402


@pytest.fixture(scope="session")
def ssd():
    """The CUDA library's binding (built in-tree first if its sources changed)."""
    from mamba_ssd_state_02_b200 import build
    build.build()
    from mamba_ssd_state_02_b200 import ssd as mod
    return mod


@pytest.fixture(scope="session")
def cuda_dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")
