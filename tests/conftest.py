import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a); parity tests of the CUDA path")


import pytest  # noqa: E402


@pytest.fixture(autouse=True)
def _fresh_device_status(request):
    """GPU tests start with the library's device error word clear, so an error
    one test provokes on purpose (or causes) is reported by that test alone."""
    if request.node.get_closest_marker("gpu") is not None:
        from sparse_mixture_experts_gating_b200 import clear_status
        clear_status()
    yield
