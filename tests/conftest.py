import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


import pytest  # noqa: E402


@pytest.fixture
def no_visible_gpu():
    """For host-side tests that hand fake device addresses to entry points and rely on the
    argument checks to refuse every call before a launch: they run only where no CUDA device
    is visible, so a regression in those checks can never launch a kernel on a fake address."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-only check: runs with no visible CUDA device")
