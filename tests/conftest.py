import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


import pytest  # noqa: E402


@pytest.fixture(autouse=True)
def _no_device_timeout(request):
    """After every GPU test: no bounded device-side wait gave up while it ran (a
    wait that gives up lets the kernel drain with undefined results, so a test
    whose tolerance happens to absorb them must still fail)."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    from chunked_state_space_b200 import ssd
    status = ssd.ssd_read_device_status()
    assert status == 0, f"a bounded device-side wait gave up during this test ({ssd.status_string(status)})"
