"""GPU W4A16 GEMM entry at M = 1..64 (tcgen05 tensor cores: the int8 decode
kernel at M <= 16 with K a multiple of 512, the bf16 skinny kernel otherwise;
the M <= 16 cases run on both) against the CPU oracle's fp64 linear:
rel-L2 <= 1e-3 and max-abs <= 1e-2 * rms(y)."""
import numpy as np
import pytest

import oracle
import post_weight_quantization_wq_b200 as wq
from post_weight_quantization_wq_b200 import inputs
from gpu_util import check_close, dev_bf16, quantize_and_check, sample_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("N,K", [(128, 128), (200, 640), (256, 1024), (384, 2048), (129, 11008),
                                 (300, 1536)])
def test_gemm_small(N, K, sym, decode_kernel):
    W = inputs.weights(N, K, 0.02, seed=3 * N + K)
    qw, P, s, z = quantize_and_check(W, None, sym)
    for M in (1, 3, 8, 16, 24, 32, 40, 48, 64):
        chans = inputs.outlier_channels(K, 0.01, seed=K)
        x = inputs.activations(M, K, seed=M + 7 * K, channels=chans, mult=30.0)
        y = wq.linear(dev_bf16(x), qw, path="gemm").cpu().numpy()
        check_close(y, oracle.linear(x, P, s, z, K, sym=sym), f"N={N} K={K} M={M}")


def test_gemm_zero_point_outside_code_range():
    """Groups whose zero point lies outside [0, 15] (all weights of one sign)."""
    N, K = 256, 1024
    w = (np.random.default_rng(4).standard_normal((N, K)) * 0.02).astype(np.float32)
    w[:64] = np.abs(w[:64]) + 0.3
    W = inputs.to_bf16_bits(w)
    qw, P, s, z = quantize_and_check(W, None, False)
    x = inputs.activations(32, K, seed=5)
    y = wq.linear(dev_bf16(x), qw, path="gemm").cpu().numpy()
    check_close(y, oracle.linear(x, P, s, z, K, sym=False))


def test_gemm_row_tile_split_across_many_ctas(decode_kernel):
    N, K = 128, 28672
    W = inputs.weights(N, K, 0.015, seed=21)
    qw, P, s, z = quantize_and_check(W, None, False)
    x = inputs.activations(16, K, seed=22)
    y = wq.linear(dev_bf16(x), qw, path="gemm").cpu().numpy()
    check_close(y, oracle.linear(x, P, s, z, K, sym=False))


def test_gemm_deterministic():
    import torch
    N, K = 1024, 8192
    W = inputs.weights(N, K, 0.015, seed=31)
    qw, *_ = quantize_and_check(W, None, False)
    x = dev_bf16(inputs.activations(64, K, seed=32))
    assert torch.equal(wq.linear(x, qw, path="gemm"), wq.linear(x, qw, path="gemm"))


@pytest.mark.parametrize("li", [0, 1])
def test_workload_batched_decode_full_size(li, decode_kernel):
    """The batched-decode workload at full size (28672x8192 and 8192x28672,
    M = 16, 32, 64, 1% activation channels x30), sampled output rows."""
    cid = 4
    wl = inputs.WORKLOADS[cid]
    lin = wl.linears[li]
    W = inputs.workload_weight(cid, li)
    qw, P, s, z = quantize_and_check(W, None, wl.sym)
    del W
    rows = sample_rows(lin.N, seed=40 + li)
    for M in wl.Ms:
        x = inputs.workload_activations(cid, li, M)
        y = wq.linear(dev_bf16(x), qw, path="gemm").cpu().numpy()
        yref = oracle.linear(x, P, s, z, lin.K, sym=wl.sym, rows=rows)
        check_close(y[:, rows], yref, f"cfg4 {lin.name} M={M}")
