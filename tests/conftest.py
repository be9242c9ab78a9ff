import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


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
def _poison_outputs(request):
    """GPU tests: every output and workspace the binding allocates starts as
    0xFF bytes (NaN for floating point), so an element that a kernel never
    writes cannot pass by holding the bytes of an earlier, identical call."""
    if "gpu" in request.keywords:
        import semi_structured_sparse_diag_b200 as nm
        nm.set_poison(True)
    yield
