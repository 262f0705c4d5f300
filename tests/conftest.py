import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")
    config.addinivalue_line("markers", "slow: long CPU test (full-size oracle)")


import pytest  # noqa: E402


@pytest.fixture(autouse=True)
def _no_silent_kernel_timeouts(request, monkeypatch):
    """GPU tests: closing a context first reads its device error word, so a
    bounded wait that gave up inside any kernel of the test fails the test
    (an aborted kernel can leave outputs that still pass a loose check)."""
    if request.node.get_closest_marker("gpu") is None:
        yield
        return
    from step_flow_map_b200 import host
    import step_flow_map_b200 as fmb
    orig = host.Context.close

    def close(self):
        if self.ctx:
            try:
                fmb.fm_device_status(self.ctx)
            finally:
                orig(self)

    monkeypatch.setattr(host.Context, "close", close)
    yield
