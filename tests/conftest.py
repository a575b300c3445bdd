import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size case (minutes)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.default()  # builds libjloracle.so if needed
    return oracle


@pytest.fixture(scope="session")
def jl():
    """The CUDA library's Python binding (requires a GPU to run kernels)."""
    import long_context_attention_bifocal_b200 as jl
    return jl
