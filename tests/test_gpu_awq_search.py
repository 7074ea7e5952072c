"""The AWQ scale search on the GPU (wq_awq_search) against the fp64 oracle
(oracle.calibrated.awq_search), "3.6 量化(Quantization)", section AWQ: for
alpha = i/20, s = s_X^alpha over its geometric mean, RTN of W diag(s), loss
||X W^T - (X / s) dequant(Q(W diag(s)))^T||^2 on the calibration rows.

Both sides compute the losses in fp64 in different summation orders (and the
GPU forms W - w_hat/s before the product), so they agree to about 1e-13
relative; the tests allow 1e-6.  The chosen alpha must be the oracle's unless
the two smallest losses are that close; its scale s must match the oracle's
fp32 s (the fp64 power and logarithm of the two math libraries can differ in
the last bit, so a channel may differ by one fp32 ulp where the fp64 value
lies on a rounding boundary; none does here)."""
import numpy as np
import pytest

from oracle import calibrated as cal
import post_weight_quantization_wq_b200 as wq
from post_weight_quantization_wq_b200 import _binding as abi
from post_weight_quantization_wq_b200 import inputs
from gpu_util import dev_bf16

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-6


def _compare(W, X, sym):
    got = wq.awq_search(dev_bf16(W), dev_bf16(X), symmetric=sym)
    ref = cal.awq_search(W, X, sym=sym)
    rel = np.abs(got["losses"] - ref["losses"]) / np.abs(ref["losses"])
    assert np.all(rel <= LOSS_RTOL), rel.max()
    if got["i"] != ref["i"]:
        a, b = ref["losses"][ref["i"]], ref["losses"][got["i"]]
        assert abs(a - b) <= LOSS_RTOL * abs(a), (got["i"], ref["i"])
    else:
        s = got["s"].cpu().numpy()
        assert np.array_equal(s.view(np.uint32), ref["s"].view(np.uint32)), \
            np.max(np.abs(s.view(np.int32).astype(np.int64) - ref["s"].view(np.int32)))
    return got, ref


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("N,K,T", [(96, 512, 128), (130, 384, 64), (64, 1024, 100)])
def test_awq_search_matches_the_oracle(N, K, T, sym):
    W = inputs.weights(N, K, 0.02, seed=N + K)
    ch = inputs.outlier_channels(K, 0.01, seed=K + 1)
    X = inputs.activations(T, K, seed=T + K, channels=ch, mult=20.0)
    _compare(W, X, sym)


def test_awq_search_on_the_decoder_layer_recipe():
    """A 256-row slice of the AWQ workload's q projection (K = 8192) with the
    workload's 128 calibration rows (1 % of channels x50)."""
    cid, li = 5, 0
    wl = inputs.WORKLOADS[cid]
    K = wl.linears[li].K
    W = inputs.workload_weight(cid, li)[:256].copy()
    X = inputs.activations(wl.calib_rows, K, inputs.calib_seed(cid, K),
                           inputs.outlier_channels(K, wl.act_outlier_frac, inputs.outlier_seed(cid, K)),
                           wl.calib_outlier_mult)
    _compare(W, X, False)


def test_awq_search_is_deterministic():
    import torch
    W = inputs.weights(256, 2048, 0.015, seed=5)
    X = inputs.activations(128, 2048, seed=6, channels=inputs.outlier_channels(2048, 0.01, 7),
                           mult=50.0)
    a = wq.awq_search(dev_bf16(W), dev_bf16(X))
    b = wq.awq_search(dev_bf16(W), dev_bf16(X))
    assert np.array_equal(a["losses"], b["losses"]) and a["i"] == b["i"]
    assert torch.equal(a["s"], b["s"])


def test_awq_search_rejects_bad_arguments():
    import torch
    buf = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    need = abi.wq_awq_search_workspace_bytes(8, 16, 256, 4)
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    args = dict(W=buf, X=buf, T=8, N=16, K=256, group_size=128, symmetric=0, n_grid=4,
                losses=buf, scale_out=buf, best=buf, workspace=ws, ws_bytes=need)
    for k, v, st in (("K", 200, abi.WQ_ERR_UNSUPPORTED_SHAPE), ("T", 0, abi.WQ_ERR_UNSUPPORTED_SHAPE),
                     ("n_grid", 0, abi.WQ_ERR_INVALID_ARG), ("best", None, abi.WQ_ERR_INVALID_ARG),
                     ("ws_bytes", need - 1, abi.WQ_ERR_WORKSPACE_TOO_SMALL)):
        a = dict(args)
        a[k] = v
        assert abi.wq_awq_search(**a) == st, k
