import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built library")


@pytest.fixture(scope="session")
def gpu_lib():
    """The CUDA library, loaded through its Python binding; fails loudly when absent."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("a gpu-marked test ran without a CUDA device")
    import sparse_moe_gemv_b200 as smg
    smg.load()
    return smg
