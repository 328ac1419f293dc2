import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes)")


@pytest.fixture(autouse=True)
def _no_device_wait_gave_up(request):
    """Every GPU test: no bounded device-side wait of the library may give up
    while it runs (such a wait ends the kernel early with partial output)."""
    if request.node.get_closest_marker("gpu") is None:
        yield
        return
    import gated_delta_rule_72_b200 as gdn
    before = gdn.gdn_device_timeouts()
    yield
    after = gdn.gdn_device_timeouts()
    assert after == before, "bounded device-side waits gave up during the test: %d" % (after - before)
