"""Failure detection without a GPU fault: with the kernels' bounded waits
cut to 1 ns, a GEMV or GEMM whose pipeline barriers are not yet satisfied
gives up, records WQ_ERR_TIMEOUT in the device error word, drains its own
copies and MMAs and returns; wq_last_device_status reports it, and with the
normal limit restored (and the workspace counters zeroed, as the header
asks after a timeout) the next call on the same context is correct."""
import numpy as np
import pytest

import oracle
import post_weight_quantization_wq_b200 as wq
from post_weight_quantization_wq_b200 import _binding as abi
from post_weight_quantization_wq_b200 import inputs
from gpu_util import check_close, dev_bf16, quantize_and_check

pytestmark = pytest.mark.gpu

DEFAULT_WAIT_NS = 2_000_000_000


@pytest.mark.parametrize("M,path", [(1, "gemv"), (4, "gemv"), (16, "gemm"), (24, "gemm")])
def test_wait_timeout_is_reported_and_context_stays_usable(M, path):
    import torch
    N, K = 4096, 8192
    W = inputs.weights(N, K, 0.015, seed=41)
    qw, P, s, z = quantize_and_check(W, None, False)
    x = inputs.activations(M, K, seed=42)
    xt = dev_bf16(x)
    need = (abi.wq_gemm_workspace_bytes if path == "gemm" else abi.wq_workspace_bytes)(M, N, K)
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda")
    assert abi.wq_last_device_status() == abi.WQ_OK
    try:
        abi.wq_debug_set_wait_limit_ns(1)
        wq.linear(xt, qw, workspace=ws, path=path)
        st = abi.wq_last_device_status()
    finally:
        abi.wq_debug_set_wait_limit_ns(DEFAULT_WAIT_NS)
    assert st == abi.WQ_ERR_TIMEOUT
    assert abi.wq_last_device_status() == abi.WQ_OK          # the word was cleared
    ws.zero_()
    y = wq.linear(xt, qw, workspace=ws, path=path).cpu().numpy()
    assert abi.wq_last_device_status() == abi.WQ_OK
    check_close(y, oracle.linear(x, P, s, z, K, sym=False), f"{path} after a timeout")


@pytest.mark.parametrize("M,path", [(1, "gemv"), (4, "gemv"), (16, "gemm"), (24, "gemm")])
def test_timeout_with_the_cached_workspace(M, path):
    """linear() without a workspace uses one cached per (device, stream).  A
    call cut short by a timeout may leave its completion counters set;
    wq.last_device_status() reports the timeout and drops the cached
    workspaces, so the next default call is correct without any manual
    zeroing."""
    N, K = 4096, 8192
    W = inputs.weights(N, K, 0.015, seed=43)
    qw, P, s, z = quantize_and_check(W, None, False)
    x = inputs.activations(M, K, seed=44)
    xt = dev_bf16(x)
    wq.linear(xt, qw, path=path)                     # creates the cached workspace
    assert wq.last_device_status() == abi.WQ_OK
    try:
        abi.wq_debug_set_wait_limit_ns(1)
        for _ in range(3):
            wq.linear(xt, qw, path=path)
        st = wq.last_device_status()
    finally:
        abi.wq_debug_set_wait_limit_ns(DEFAULT_WAIT_NS)
    assert st == abi.WQ_ERR_TIMEOUT
    yref = oracle.linear(x, P, s, z, K, sym=False)
    for _ in range(2):
        y = wq.linear(xt, qw, path=path).cpu().numpy()
        assert wq.last_device_status() == abi.WQ_OK
        check_close(y, yref, f"{path} with the cached workspace after a timeout")
