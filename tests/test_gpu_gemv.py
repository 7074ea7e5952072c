"""GPU W4A16 GEMV (M = 1..8) against the CPU oracle's fp64 linear on the same
seeded inputs: rel-L2 <= 1e-3 and max-abs <= 1e-2 * rms(y)."""
import numpy as np
import pytest

import oracle
import post_weight_quantization_wq_b200 as wq
from post_weight_quantization_wq_b200 import inputs
from gpu_util import (check_close, dev_bf16, dev_f32, quantize_and_check, sample_rows)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("N,K", [(1, 128), (200, 640), (256, 1024), (130, 1408), (384, 2048),
                                 (129, 11008), (1, 512), (200, 1536), (129, 5120)])
def test_gemv_small_all_m(N, K, sym, decode_kernel):
    W = inputs.weights(N, K, 0.02, seed=N + K)
    qw, P, s, z = quantize_and_check(W, None, sym)
    for M in range(1, 9):
        x = inputs.activations(M, K, seed=M * 31 + K)
        y = wq.linear(dev_bf16(x), qw, path="gemv").cpu().numpy()
        yref = oracle.linear(x, P, s, z, K, sym=sym)
        check_close(y, yref, f"N={N} K={K} M={M}")


@pytest.mark.parametrize("M", [1, 2, 3, 4])
def test_gemv_row_tile_split_across_many_ctas(M, decode_kernel):
    """N = 128 with K = 28672: one row tile of 56 slabs, more CTAs than a row
    tile has slabs, so every CTA holds a piece and the last one adds them."""
    N, K = 128, 28672
    W = inputs.weights(N, K, 0.015, seed=7)
    qw, P, s, z = quantize_and_check(W, None, False)
    x = inputs.activations(M, K, seed=8)
    y = wq.linear(dev_bf16(x), qw, path="gemv").cpu().numpy()
    check_close(y, oracle.linear(x, P, s, z, K, sym=False))


@pytest.mark.parametrize("M", [1, 2, 3, 4, 8])
def test_gemv_awq_fold_small(M, decode_kernel):
    N, K = 256, 1536
    W = inputs.weights(N, K, 0.015, seed=91)
    chans = inputs.outlier_channels(K, 0.01, seed=92)
    X = inputs.bf16_bits_to_f32(inputs.activations(128, K, seed=93, channels=chans, mult=50.0))
    s = inputs.awq_scale_from_calibration(X)
    qw, P, sc, z = quantize_and_check(W, s, False)
    x = inputs.activations(M, K, seed=94, channels=chans, mult=50.0)
    inv = (1.0 / s).astype(np.float32)
    y = wq.linear(dev_bf16(x), qw, inv_act_scale=dev_f32(inv), path="gemv").cpu().numpy()
    yref = oracle.linear(x, P, sc, z, K, sym=False, awq_s=s)
    check_close(y, yref, f"awq M={M}")


def test_gemv_nonfinite_group_gives_nan_rows(decode_kernel):
    N, K = 64, 1024
    w = (np.random.default_rng(1).standard_normal((N, K)) * 0.02).astype(np.float32)
    w[9, 300] = np.inf
    W = inputs.to_bf16_bits(w)
    qw, P, s, z = quantize_and_check(W, None, False)
    x = inputs.activations(1, K, seed=3)
    y = wq.linear(dev_bf16(x), qw, path="gemv").cpu().numpy()
    yref = oracle.linear(x, P, s, z, K, sym=False)
    assert np.isnan(y[0, 9]) and np.isnan(yref[0, 9])
    keep = np.arange(N) != 9
    check_close(y[:, keep], yref[:, keep])


def test_gemv_deterministic_and_workspace_reuse(decode_kernel):
    """Bit-identical reruns; one workspace shared by calls of different sizes
    (the completion counters are left at zero by every call)."""
    import torch
    shapes = [(1024, 8192, 1), (512, 4096, 3), (1024, 8192, 8), (256, 1024, 2)]
    ws = torch.zeros(max(wq._binding.wq_workspace_bytes(M, N, K) for N, K, M in shapes),
                     dtype=torch.uint8, device="cuda")
    for N, K, M in shapes:
        W = inputs.weights(N, K, 0.02, seed=N + 3 * K)
        qw, P, s, z = quantize_and_check(W, None, False)
        x = dev_bf16(inputs.activations(M, K, seed=K + M))
        y1 = wq.linear(x, qw, workspace=ws, path="gemv")
        y2 = wq.linear(x, qw, workspace=ws, path="gemv")
        assert torch.equal(y1, y2)
        yref = oracle.linear(x.cpu().view(torch.int16).numpy().view(np.uint16), P, s, z, K,
                             sym=False)
        check_close(y1.cpu().numpy(), yref)
    assert int(ws[:wq._binding.WQ_WORKSPACE_COUNTER_BYTES].count_nonzero()) == 0


@pytest.mark.parametrize("N,K", [(1, 2048), (64, 1664), (100, 3200), (128, 3584), (600, 1024)])
def test_gemv_small_grid_finishes_every_row_tile(N, K, decode_kernel):
    """Tile counts one more than a multiple of three at M = 1 (three teams per
    CTA): a grid with two teams more than tiles would leave a team without
    tiles among a row tile's owners, and that row tile's split-K sum would
    never be finished.  Every row must come out right and the completion
    counters must be left at zero."""
    import torch
    W = inputs.weights(N, K, 0.02, seed=N + 5 * K)
    qw, P, s, z = quantize_and_check(W, None, False)
    ws = torch.zeros(max(wq._binding.wq_workspace_bytes(1, N, K), 16), dtype=torch.uint8,
                     device="cuda")
    x = inputs.activations(1, K, seed=K + 1)
    for _ in range(2):
        y = wq.linear(dev_bf16(x), qw, workspace=ws, path="gemv").cpu().numpy()
        check_close(y, oracle.linear(x, P, s, z, K, sym=False), f"N={N} K={K}")
        assert int(ws[:wq._binding.WQ_WORKSPACE_COUNTER_BYTES].count_nonzero()) == 0


# ----------------------------------------------------------------- full sizes

FULL = [(cid, li) for cid in (1, 2, 3, 5) for li in range(len(inputs.WORKLOADS[cid].linears))]


@pytest.mark.parametrize("cid,li", FULL)
def test_workload_full_size(cid, li):
    """Every linear of the single-linear, Llama-7B, Llama-70B and AWQ-layer
    workloads at full size: bit-exact quantization and layout, then the GEMV
    at each of the workload's M values on sampled output rows (tile edges
    included)."""
    wl = inputs.WORKLOADS[cid]
    lin = wl.linears[li]
    W = inputs.workload_weight(cid, li)
    s_awq = inputs.workload_awq_scale(cid, li)
    qw, P, s, z = quantize_and_check(W, s_awq, wl.sym)
    del W
    inv = None if s_awq is None else dev_f32((1.0 / s_awq).astype(np.float32))
    rows = sample_rows(lin.N, seed=cid * 10 + li)
    for M in wl.Ms:
        x = inputs.workload_activations(cid, li, M)
        y = wq.linear(dev_bf16(x), qw, inv_act_scale=inv, path="gemv").cpu().numpy()
        yref = oracle.linear(x, P, s, z, lin.K, sym=wl.sym, awq_s=s_awq, rows=rows)
        check_close(y[:, rows], yref, f"cfg{cid} {lin.name} M={M}")


@pytest.mark.parametrize("sym", [False, True])
def test_headline_linear_both_kernels(sym, decode_kernel):
    """8192 x 28672 (the down projection of a Llama-70B-shaped layer) at
    M = 1, 2, 3, 4, 5, 8 on both decode kernels, sampled rows against the
    oracle."""
    N, K = 8192, 28672
    W = inputs.weights(N, K, 0.015, seed=123 + sym)
    qw, P, s, z = quantize_and_check(W, None, sym)
    del W
    rows = sample_rows(N, seed=17)
    for M in (1, 2, 3, 4, 5, 8):
        x = inputs.activations(M, K, seed=40 + M)
        y = wq.linear(dev_bf16(x), qw, path="gemv").cpu().numpy()
        yref = oracle.linear(x, P, s, z, K, sym=sym, rows=rows)
        check_close(y[:, rows], yref, f"{decode_kernel} sym={sym} M={M}")
