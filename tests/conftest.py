import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the CUDA library")


GOLDEN = os.path.join(ROOT, "tests", "golden")


@pytest.fixture(scope="session")
def libmoe_path():
    """Builds libmoe.so in-tree if it is missing or older than its sources."""
    from routing_dispatch_expert_fp32_b200 import build
    return build.build()


@pytest.fixture(scope="session")
def moe(libmoe_path):
    """The ctypes binding (GPU tests only call compute entry points)."""
    from routing_dispatch_expert_fp32_b200 import moe as m
    return m
