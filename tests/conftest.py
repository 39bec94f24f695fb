import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA device (B200); parity of the CUDA path against the oracle")


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA library through its Python binding.  On a machine with a GPU a
    missing or unloadable library is an error, never a skip."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device on this machine")
    import relu_linear_attention_attn_b200 as sla
    sla.load()  # raises if the shared library is missing
    return sla
