import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def full_layer():
    """The whole H=6144, I=2048, E=256 layer on the GPU with its per-expert oracle cache,
    built once and shared by every module's full-size tests."""
    import bit_quantized_moe_nvfp4_b200 as nv
    from helpers import FullLayer
    return FullLayer(nv)
