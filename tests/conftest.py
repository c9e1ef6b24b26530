import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


@pytest.fixture(autouse=True)
def _guarded_outputs(request):
    """GPU tests: every output the binding allocates, and every output a test
    makes with guard.empty, sits between sentinel bytes that must be
    unchanged when the test ends (out-of-bounds writes fail the test)."""
    if request.node.get_closest_marker("gpu") is None:
        yield
        return
    import guard
    with guard.session(), guard.binding_allocations():
        yield
