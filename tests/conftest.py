import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The built CUDA library, loaded through the Python binding (GPU tests only)."""
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_linear_attention_ttt_b200 as ttt

    ttt.load_library()
    return ttt


@pytest.fixture
def tuning(cuda_lib):
    """set(key, value) for the library's kernel-variant choices; every choice goes back to the
    automatic one when the test ends."""
    cuda_lib.reset_tuning()
    yield cuda_lib.set_tuning
    cuda_lib.reset_tuning()
