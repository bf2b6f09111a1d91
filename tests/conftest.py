"""Shared pytest configuration.

Tests marked ``gpu`` need a CUDA device (a B200) and call the CUDA library
through its C ABI; everything else runs on the CPU (oracle pins, host-side
logic, library symbol checks)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built CUDA library")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def fpq():
    """The CUDA library's Python binding.  GPU tests fail (never skip) when
    the device or the built library is missing: there is no fallback."""
    import torch
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"
    import mxfp8_block_scaled_warp_b200 as lib
    lib.load()
    return lib
