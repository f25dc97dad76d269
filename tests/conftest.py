import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built libnslm.so")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


import pytest  # noqa: E402


@pytest.fixture(autouse=True)
def _guards_intact(request):
    """After every GPU test: no kernel wrote into the guard regions around the
    buffers the test took from tests/guard.py."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import torch

    import guard
    if torch.cuda.is_available():
        guard.check_all()
    else:
        guard.forget()
