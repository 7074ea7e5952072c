"""The Python layer refuses inputs the C ABI would misread (it only sees raw
pointers): host tensors, other dtypes, strided views, wrong shapes.  All
checks run before any CUDA call, so they are tested on the CPU."""
import pytest
import torch

import post_weight_quantization_wq_b200 as wq


def _fake_qw(N=256, K=1024):
    # a QuantizedWeight whose buffers are CPU tensors: linear() must refuse x
    # before it looks at them
    return wq.QuantizedWeight(N, K, False, None, None, None, torch.empty(16, dtype=torch.uint8))


def test_quantize_refuses_host_and_wrong_dtype():
    with pytest.raises(ValueError, match="CUDA"):
        wq.quantize(torch.zeros(4, 128, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="2-D"):
        wq.quantize(torch.zeros(128, dtype=torch.bfloat16))


def test_linear_refuses_host_x():
    with pytest.raises(ValueError, match="CUDA"):
        wq.linear(torch.zeros(1, 1024, dtype=torch.bfloat16), _fake_qw())
    with pytest.raises(ValueError, match="2-D"):
        wq.linear(torch.zeros(1024, dtype=torch.bfloat16), _fake_qw())


def test_require_messages():
    from post_weight_quantization_wq_b200 import _require
    with pytest.raises(TypeError):
        _require([1, 2], "x", torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        _require(torch.zeros(2, 2), "x", torch.float32)
