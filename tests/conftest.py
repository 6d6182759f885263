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
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU in this environment")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(params=[0, 1], ids=["scan_cluster", "fused"])
def decode_kernel(request):
    """Run a decode-path test under both decode kernels (the index scan +
    per-row cluster kernels, and the fused single-launch kernel)."""
    import compressed_sparse_attention_topk_b200 as csa2
    prev = csa2.get_decode_kernel()
    csa2.set_decode_kernel(request.param)
    yield request.param
    csa2.set_decode_kernel(prev)
