import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def gpu_lib():
    """The CUDA library, built in-tree if stale; a GPU test without a CUDA device fails loudly."""
    import torch
    from deformable_slide_attention_b200 import abi, build
    build.build()
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"
    assert abi.dsa3d_abi_version() == 3
    return abi
