import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity cases")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def moe():
    """The CUDA library's Python binding, built in-tree first (nvcc only;
    no GPU needed to build or load)."""
    from quantized_routed_expert_top_b200 import build
    build.build()
    import quantized_routed_expert_top_b200 as m
    m.lib()
    return m
