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


@pytest.fixture(params=["fused", "multi_kernel", "cluster"])
def decode_mode(request):
    """Run a decode-step test under each step implementation: the fused step
    (selection + attention in one persistent kernel), the multi-kernel step
    and the cluster step (one kernel per step where the sizes fit a
    thread-block cluster; other sizes fall back to the multi-kernel step).
    The process-wide mode is restored afterwards."""
    from hash_aware_top_hata_b200 import hata as H
    mode = {"fused": H.HATA_MODE_FUSED, "multi_kernel": H.HATA_MODE_MULTI_KERNEL,
            "cluster": H.HATA_MODE_CLUSTER}[request.param]
    H.hata_set_decode_mode(mode)
    yield request.param
    H.hata_set_decode_mode(H.HATA_MODE_AUTO)
