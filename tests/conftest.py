import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    # A GPU test on a machine without CUDA fails loudly instead of skipping:
    # selecting -m gpu on a box with no GPU is a setup error, not a pass.
    pass


@pytest.fixture(scope="session")
def cuda_lib():
    """The built CUDA library's Python binding; fails loudly when unavailable."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test selected but torch.cuda.is_available() is False")
    import long_context_decode_swa_b200 as rswa
    rswa.load()  # raises if librswa.so is missing
    return rswa
