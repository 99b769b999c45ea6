import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes)")


@pytest.fixture(scope="session", autouse=True)
def _launch_overlap_default():
    """With NVFP4_TEST_LAUNCH_OVERLAP=1 every GPU test runs with launch overlap on."""
    from tests import _helpers as H
    if H.LAUNCH_OVERLAP_DEFAULT:
        import nvfp4_w4a4_quantized_quantizer_b200 as nv
        nv.nvfp4_set_launch_overlap(True)
    yield


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)
