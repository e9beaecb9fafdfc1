import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))
for p in (ROOT, HERE):
    if p not in sys.path:
        sys.path.insert(0, p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity cases (minutes)")


import pytest  # noqa: E402


@pytest.fixture(autouse=True)
def _fresh_prefill_auto_state(request):
    """The default prefill mode switches a device to adaptive P once a launch meets inputs
    that make many rows sharp, for every later launch in the process. Each GPU test starts
    and ends with the switch off, so that it runs the kernel its inputs choose."""
    gpu = request.node.get_closest_marker("gpu") is not None
    if gpu:
        import sliding_window_causal_b200 as swa
        swa.prefill_auto_state(clear=True)
    yield
    if gpu:
        swa.prefill_auto_state(clear=True)
