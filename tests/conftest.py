import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def lib():
    """The CUDA library through its C ABI (fails loudly if it is not built)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_weight_only_linear_b200 import awq, build
    build.build()
    awq.load_library()
    return awq
