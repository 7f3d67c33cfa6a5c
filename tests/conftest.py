import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def golden_lines(name):
    """Non-comment, non-empty lines of a fixture under tests/golden/."""
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.lstrip().startswith("#")]


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA path's binding; skips nothing -- a GPU test without it fails."""
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import ternary_bit_linear_b200 as tq

    tq.load()
    return tq
