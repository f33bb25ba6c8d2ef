import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running test")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(params=[1, 0], ids=["two_kernels", "fused"])
def bwd_kernels(request):
    """Runs a backward test with each backward path: 1 the two kernels (the
    default), 0 the fused kernel (dQ by reductions); the switch is restored."""
    from ring_ulysses_sequence_b200 import native
    before = native.rm_get_bwd_deterministic()
    native.rm_set_bwd_deterministic(request.param)
    yield request.param
    native.rm_set_bwd_deterministic(before)
