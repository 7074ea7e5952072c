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


@pytest.fixture(params=["int8_tc", "int8_off"])
def decode_kernel(request):
    """Runs a linear test once per decode kernel: the default choice (the
    int8 tensor-core kernel where it applies: wq_gemv_w4a16 at M = 2..8 and
    wq_gemm_w4a16 at M <= 16, K a multiple of 512) and with that kernel
    switched off (the CUDA-core GEMV, the bf16 tensor-core GEMM)."""
    from post_weight_quantization_wq_b200 import _binding as abi
    abi.wq_debug_gemv_force_cuda_cores(int(request.param == "int8_off"))
    try:
        yield request.param
    finally:
        abi.wq_debug_gemv_force_cuda_cores(0)
