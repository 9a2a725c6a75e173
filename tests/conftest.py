import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    # GPU tests cannot run without a device; skip them (instead of failing) on CPU hosts
    # when they were not deselected with -m "not gpu".
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device on this host")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(params=[1, 2, 3], ids=["segments", "per_group", "per_group_4warps"])
def bwd_path(request):
    """Runs a backward test on both reverse passes of the TMA path: the time-parallel
    segments (1) and one CTA per channel group (2), whatever the automatic choice for the
    shape would be; back to automatic (0) afterwards."""
    import rwkv_linear_attention_wkv_b200 as W
    assert W.lib.wkv_testing_set_backward_path(request.param) == 0
    yield request.param
    W.lib.wkv_testing_set_backward_path(0)
