"""The largest shapes the ABI accepts (N or K = 2^20 = WQ_MAX_DIM), through
quantize, relayout and both linears, against the CPU oracle: bit-exact
metadata and codes, y within the tolerance.  K = 2^20 is 2048 slabs of one
row tile (every team holds a piece of the same row tile); N = 2^20 is 8192
row tiles of one slab (no split-K)."""
import numpy as np
import pytest

import oracle
import post_weight_quantization_wq_b200 as wq
from post_weight_quantization_wq_b200 import _binding as abi
from post_weight_quantization_wq_b200 import inputs
from gpu_util import check_close, dev_bf16, quantize_and_check

pytestmark = pytest.mark.gpu

MAXD = 1 << 20


@pytest.mark.parametrize("N,K", [(128, MAXD), (MAXD, 128)])
def test_max_dims_gemv_and_gemm(N, K):
    W = inputs.weights(N, K, 0.02, seed=N + 3)
    qw, P, s, z = quantize_and_check(W, None, False)
    for M, path in ((1, "gemv"), (3, "gemm"), (16, "gemm")):
        x = inputs.activations(M, K, seed=M + 5)
        y = wq.linear(dev_bf16(x), qw, path=path).cpu().numpy()
        rows = None if N <= 4096 else np.sort(np.random.default_rng(7).choice(N, 2048, replace=False))
        yref = oracle.linear(x, P, s, z, K, sym=False, rows=rows)
        check_close(y if rows is None else y[:, rows], yref, f"{path} N={N} K={K} M={M}")
    assert wq.last_device_status() == 0


def test_dims_above_the_maximum_are_refused():
    assert abi.wq_packed_bytes(MAXD + 1, 128, 128, 0, 1) == 0
    assert abi.wq_packed_bytes(128, MAXD + 128, 128, 0, 1) == 0
