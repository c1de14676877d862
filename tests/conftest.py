import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(autouse=True)
def _output_guards(request):
    """After every GPU test: the guard regions around its output buffers
    (tests/helpers.py: guarded) must be intact."""
    yield
    if request.node.get_closest_marker("gpu") is not None:
        import helpers
        helpers.check_guards()
