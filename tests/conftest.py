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


@pytest.fixture(scope="session")
def hooked(libmoe_path):
    """A test-only build of the library (never the shipped one) compiled with
    MOE_TEST_HOOKS and 20 ms pipeline waits: moe_test_hooks(stall, max_ctas)
    makes the tcgen05 GEMM producers issue no loads, or caps the GEMM grid.
    Returns the ctypes handle with the binding's signatures; the hooks are
    switched off again at the end of the session."""
    import ctypes
    from routing_dispatch_expert_fp32_b200 import build
    from routing_dispatch_expert_fp32_b200 import moe as m
    path = build.build(extra=["-DMOE_TEST_HOOKS", "-DMOE_WAIT_LIMIT_NS=20000000ull"],
                       out=os.path.join(ROOT, "_build", "libmoe_test_hooks.so"))
    lib = ctypes.CDLL(path)
    for name, (args, res) in m._SIGS.items():
        f = getattr(lib, name)
        f.argtypes, f.restype = args, res
    lib.moe_test_hooks.argtypes = [ctypes.c_int, ctypes.c_int]
    lib.moe_test_hooks.restype = ctypes.c_int
    yield lib
    lib.moe_test_hooks(0, 0)
