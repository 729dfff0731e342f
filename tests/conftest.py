import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")
    config.addinivalue_line("markers", "slow: long CPU test")


def gpu_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def golden():
    def read(name):
        out = {}
        with open(os.path.join(ROOT, "tests", "golden", name)) as f:
            for line in f:
                line = line.strip()
                if not line or line.startswith("#"):
                    continue
                k, *v = line.split()
                out[k] = v
        return out
    return read
