import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA B200 (runs the sm_100a library)")


@pytest.fixture(scope="session")
def cuda():
    """GPU tests never skip silently: without a device they fail."""
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("gpu-marked test run without a CUDA device")
    return torch.device("cuda:0")


def read_golden(name):
    vals = {}
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split()[:2]
            vals[k] = float(v)
    return vals
