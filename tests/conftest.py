import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU check")


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


@pytest.fixture(params=["tensor_cores", "cuda_cores"])
def gemv_kernel(request):
    """Runs a GEMV test once per decode kernel: the default choice (the
    integer tensor-core kernel where it applies: M = 2..8, K a multiple of
    512) and the CUDA-core kernel forced for every shape."""
    from post_weight_quantization_wq_b200 import _binding as abi
    abi.wq_debug_gemv_force_cuda_cores(int(request.param == "cuda_cores"))
    try:
        yield request.param
    finally:
        abi.wq_debug_gemv_force_cuda_cores(0)
