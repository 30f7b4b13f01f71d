import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running (full-size workloads)")


@pytest.fixture
def golden_dir():
    return GOLDEN


def read_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [line.rstrip("\n") for line in f if line.strip() and not line.startswith("#")]
