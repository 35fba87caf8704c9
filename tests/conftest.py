import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built libisd.so")


@pytest.fixture(scope="session")
def cuda_lib():
    """The product library on a GPU (fails loudly if it is missing)."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test collected on a machine without a GPU")
    from strided_verify_propose_b200 import binding
    return binding.lib()
