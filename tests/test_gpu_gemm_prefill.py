"""wq_gemm_w4a16 with many activation rows (the prefill kernel: tiles of 128
weight rows x up to 128 activation rows, dequantized bf16 weights in shared
memory, running sums in tensor memory), against the oracle's fp64 linear:
rel-L2 <= 1e-3 and max-abs <= 1e-2 rms(y) ("大模型量化全景解析", section 八:
prefill is compute-bound; the same W4A16 product as decode)."""
import numpy as np
import pytest

import oracle
import post_weight_quantization_wq_b200 as wq
from post_weight_quantization_wq_b200 import _binding as abi
from post_weight_quantization_wq_b200 import inputs
from gpu_util import check_close, dev_bf16, quantize_and_check, sample_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("N,K", [(256, 1024), (200, 1408), (129, 640)])
@pytest.mark.parametrize("M", [65, 128, 129, 300])
def test_prefill_small(N, K, M, sym):
    W = inputs.weights(N, K, 0.02, seed=N + 7 * K)
    qw, P, s, z = quantize_and_check(W, None, sym)
    ch = inputs.outlier_channels(K, 0.01, seed=K)
    x = inputs.activations(M, K, seed=M + K, channels=ch, mult=30.0)
    y = wq.linear(dev_bf16(x), qw, path="gemm").cpu().numpy()
    check_close(y, oracle.linear(x, P, s, z, K, sym=sym), f"prefill N={N} K={K} M={M}")


@pytest.mark.parametrize("M", [1, 3, 16, 33, 64])
def test_prefill_kernel_at_decode_sizes(M):
    """The many-row kernel forced on the skinny shapes (the test hook), against
    the oracle: both kernels must be right wherever they can run."""
    N, K = 384, 2048
    W = inputs.weights(N, K, 0.015, seed=M + 100)
    qw, P, s, z = quantize_and_check(W, None, False)
    x = inputs.activations(M, K, seed=M + 101)
    try:
        abi.wq_debug_gemm_force_fold(1)
        y = wq.linear(dev_bf16(x), qw, path="gemm").cpu().numpy()
    finally:
        abi.wq_debug_gemm_force_fold(0)
    check_close(y, oracle.linear(x, P, s, z, K, sym=False), f"forced M={M}")


def test_prefill_deterministic():
    import torch
    W = inputs.weights(1024, 4096, 0.015, seed=3)
    qw, P, s, z = quantize_and_check(W, None, False)
    x = dev_bf16(inputs.activations(256, 4096, seed=4))
    a = wq.linear(x, qw, path="gemm")
    b = wq.linear(x, qw, path="gemm")
    assert torch.equal(a, b)


@pytest.mark.parametrize("li,M", [(0, 512), (1, 256)])
def test_prefill_full_size(li, M):
    """The batched-decode workload's shapes (28672x8192, 8192x28672, 1 % of
    the activation channels x30) at prefill sizes: sampled output rows."""
    cid = 4
    lin = inputs.WORKLOADS[cid].linears[li]
    W = inputs.workload_weight(cid, li)
    qw, P, s, z = quantize_and_check(W, None, False)
    del W
    ch = inputs.outlier_channels(lin.K, 0.01, inputs.outlier_seed(cid, lin.K))
    x = inputs.activations(M, lin.K, seed=M + li, channels=ch, mult=30.0)
    y = wq.linear(dev_bf16(x), qw, path="gemm").cpu().numpy()
    rows = sample_rows(lin.N, n=128, seed=li)
    check_close(y[:, rows], oracle.linear(x, P, s, z, lin.K, sym=False, rows=rows),
                f"prefill {lin.N}x{lin.K} M={M}")


def test_prefill_then_skinny_on_one_workspace():
    """linear() keeps one workspace per stream for every path; the many-row
    kernel must leave the skinny kernel's completion counters (the first
    WQ_WORKSPACE_COUNTER_BYTES) at zero, so a decode-size call after a
    prefill-size one is still right."""
    N, K = 200, 640
    W = inputs.weights(N, K, 0.02, seed=3 * N + K)
    qw, P, s, z = quantize_and_check(W, None, False)
    for M in (300, 1, 16, 129, 40):
        x = inputs.activations(M, K, seed=M)
        y = wq.linear(dev_bf16(x), qw, path="gemm").cpu().numpy()
        check_close(y, oracle.linear(x, P, s, z, K, sym=False), f"shared workspace M={M}")
