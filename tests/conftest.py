import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def oracle():
    from oracle.oracle import default_oracle
    return default_oracle()


@pytest.fixture(scope="session")
def moe_lib():
    """The C-ABI library, built from source if missing or stale."""
    from top_routing_grouped_softmax_b200 import _build
    _build.build_library()
    import top_routing_grouped_softmax_b200 as moe
    return moe.lib()
