import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU and the built libqfp4 CUDA library")


def pytest_collection_modifyitems(config, items):
    """GPU tests are skipped, not failed, on a machine without a GPU."""
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(autouse=True)
def _output_guard_bands():
    """After each test, the guard bands around every guarded GPU output
    (tests/gpu_util.guarded) must be intact."""
    yield
    gu = sys.modules.get("gpu_util")
    if gu is not None:
        gu.check_guards()
