import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


@pytest.fixture(autouse=True)
def _device_index_checks(request):
    """SSM_DEBUG_CHECKS=1 (SSM_LIBRARY naming the -DSSM_DEBUG build): a GPU
    test must leave no failed device index check behind."""
    yield
    if os.environ.get("SSM_DEBUG_CHECKS") != "1" or "gpu" not in request.keywords:
        return
    import selective_state_space_35_b200 as ssm
    rep = ssm.debug_report(reset=True)
    assert rep["failures"] == 0, f"device index check failed: {rep}"
