import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size case (seconds to minutes)")


@pytest.fixture(scope="session")
def gpu():
    """The CUDA binding, loaded; skips nothing: a gpu-marked test on a box without the built
    library or without a device fails loudly."""
    import torch
    import transformer_norm_rope_b200 as gn

    assert torch.cuda.is_available(), "gpu test needs a CUDA device"
    gn.load()
    return gn
