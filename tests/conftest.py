import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs an NVIDIA B200 (sm_100a) GPU")


@pytest.fixture(scope="session")
def cuda_lib():
    """libhstu_attn.so, rebuilt first if any source is newer than it."""
    from hstu_pointwise_attention_jagged_b200 import build, binding
    build.build()
    return binding.load_library()


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.default()
