import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes)")


import pytest  # noqa: E402


@pytest.fixture(autouse=True)
def _device_status_clean(request):
    """Every GPU test must leave the sticky device status clear: a bounded wait
    that ran out inside a kernel is a failure even when the outputs compare
    equal.  (The timeout test sets and clears the status on purpose.)"""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    from scaled_dot_product_bwd_b200 import sdpa_read_device_status
    status = sdpa_read_device_status()
    assert status == 0, f"device status {status} after {request.node.nodeid}"
