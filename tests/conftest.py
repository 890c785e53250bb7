import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload, minutes of host work")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


FFN_TILINGS = {"auto": 0, "single": 1, "pair": 2}  # moe_set_ffn_tiling modes


@pytest.fixture
def ffn_tiling(request):
    """Force the bf16 FFN tile shape for one test (indirect parameter), back to auto afterwards."""
    from token_dispatch_combine_b200 import moe_set_ffn_tiling
    moe_set_ffn_tiling(FFN_TILINGS[request.param])
    yield request.param
    moe_set_ffn_tiling(0)
