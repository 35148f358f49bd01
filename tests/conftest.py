import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built libfa.so")


import pytest  # noqa: E402


@pytest.fixture(scope="session")
def fa_lib():
    """The built libfa.so (built in-tree first if it is missing)."""
    from exact_io_aware_96_b200 import build, fa
    if not os.path.exists(fa.LIB_PATH):
        build.build()
    return fa.lib()
