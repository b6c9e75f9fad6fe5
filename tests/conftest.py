import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def O():
    """The CPU oracle (built on first use)."""
    from oracle import oracle
    return oracle


@pytest.fixture(scope="session")
def cuda_lib():
    """libpagedattn.so through its binding, on a CUDA device.  Fails loudly if the library is missing."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from pagedattention_block_table_b200 import build, binding
    build.build()
    binding.lib()
    return binding
