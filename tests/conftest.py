import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle


@pytest.fixture(scope="session")
def fb():
    """The CUDA library (fails loudly if it is missing or no GPU is visible)."""
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from blockwise_scaled_fp8_fp8bw_b200 import build
    build.build()
    import blockwise_scaled_fp8_fp8bw_b200 as lib
    lib.fp8bw_init(torch.cuda.current_device())
    return lib
