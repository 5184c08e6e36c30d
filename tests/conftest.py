import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (runs the CUDA path through the C ABI)")


@pytest.fixture(scope="session")
def cuda():
    """The CUDA device for GPU tests. A GPU test never skips silently: no device is an error."""
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("GPU test selected but torch.cuda.is_available() is False")
    return torch.device("cuda:0")
