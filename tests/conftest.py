import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def has_cuda():
    import torch
    return torch.cuda.is_available()


@pytest.fixture(autouse=True)
def _index_checks(request):
    """Under M3_DEBUG_BOUNDS=1 (the index-checked library): every GPU test
    starts from a cleared record of failed index checks and fails if its
    kernels recorded any."""
    if os.environ.get("M3_DEBUG_BOUNDS") != "1" or request.node.get_closest_marker("gpu") is None:
        yield
        return
    import torch
    if not torch.cuda.is_available():
        yield
        return
    import selective_state_space_m3_b200 as m3
    m3.m3_debug_bounds_report(clear=True)
    yield
    r = m3.m3_debug_bounds_report(clear=True)
    assert r["enabled"] == 1, r
    assert r["failures"] == 0, f"failed index checks: {r}"
