import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes)")


GOLDEN = os.path.join(ROOT, "tests", "golden")


@pytest.fixture(scope="session")
def golden_dir():
    return GOLDEN


@pytest.fixture(scope="session")
def fg_lib():
    """The CUDA library's binding; raises if the library is missing (no CPU path)."""
    import torch

    import bit_compressed_decode_b200 as m
    if not torch.cuda.is_available():
        raise RuntimeError("GPU tests need a CUDA device")
    return m
