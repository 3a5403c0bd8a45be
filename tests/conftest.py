import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity case")


@pytest.fixture(autouse=True)
def _checked_build_status():
    """Under the checked build (JAMBA_CHECKED=1) the device status word is read
    after every test: an index check that fired fails the test."""
    yield
    if os.environ.get("JAMBA_CHECKED", "0") == "1":
        import torch
        if torch.cuda.is_available():
            import mamba_selective_scan_mixer_b200 as J
            J.device_status()
