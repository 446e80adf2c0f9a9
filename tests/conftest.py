import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity cases (minutes)")


@pytest.fixture(scope="session")
def oracle():
    import oracle as orc
    return orc.default()


@pytest.fixture(scope="session")
def cuda_lib():
    """The built CUDA library (built here if missing or stale)."""
    from memory_bound_cnn_wtconv_b200 import build as b
    b.build()
    import memory_bound_cnn_wtconv_b200 as w
    return w.load_library()
