import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


@pytest.fixture
def golden():
    return load_golden


def cuda_present() -> bool:
    """True when a CUDA device is visible.  Host-side tests that hand fake device pointers to
    an entry point make the calls that would pass validation only when this is False: with
    a device present such a call would launch kernels on addresses that do not exist."""
    try:
        import torch

        return torch.cuda.is_available()
    except Exception:  # pragma: no cover
        return False
