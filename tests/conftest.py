import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200 / sm_100a)")
    config.addinivalue_line("markers", "slow: full-size case (minutes of oracle time)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA library, loaded through its binding; tests needing it are marked gpu."""
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hstu_attention_b200 as hb

    hb.load()   # raises loudly if the shared library is missing
    return hb
