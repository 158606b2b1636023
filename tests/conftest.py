import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU in this environment")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(params=["fused", "multi_kernel"])
def decode_mode(request):
    """Run a decode-step test under both step implementations: the fused
    step (selection + attention in one persistent kernel) and the
    multi-kernel step.
    The process-wide mode is restored afterwards."""
    from hash_aware_top_hata_b200 import hata as H
    mode = H.HATA_MODE_FUSED if request.param == "fused" else H.HATA_MODE_MULTI_KERNEL
    H.hata_set_decode_mode(mode)
    yield request.param
    H.hata_set_decode_mode(H.HATA_MODE_AUTO)
