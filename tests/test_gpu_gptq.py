"""GPTQ on the GPU (wq_gptq_quantize) against the fp64 oracle
(oracle.calibrated.gptq_quantize, the textbook column-by-column update with
the restricted inverse Hessian), "3.6 量化(Quantization)", section GPTQ.

Integer outputs are compared bit for bit: codes, fp16 scales and zeros.  The
two sides run the same fp64 algorithm in different forms (the oracle inverts
H[j:, j:] for every column, the GPU uses one Cholesky factorization), so they
agree to about 1e-13 relative; a code can only differ where the oracle's
quotient lies that close to a rounding tie, which these seeded inputs do not
produce.  At sizes the oracle cannot finish quickly, properties that hold at
any size are checked instead: the codes decode to weights whose output error
on the calibration inputs is below plain RTN's, runs are bit-identical, and
the status word reports a Hessian that is not positive definite."""
import numpy as np
import pytest

import oracle
from oracle import calibrated as cal
import post_weight_quantization_wq_b200 as wq
from post_weight_quantization_wq_b200 import _binding as abi
from post_weight_quantization_wq_b200 import inputs
from gpu_util import dev_bf16, host_u16, host_u32

pytestmark = pytest.mark.gpu


def _gptq_gpu(W, X, sym, damp=0.01):
    qw = wq.gptq_quantize(dev_bf16(W), dev_bf16(X), symmetric=sym, damp=damp)
    return qw


def _compare_with_oracle(W, X, sym):
    N, K = W.shape
    qw = _gptq_gpu(W, X, sym)
    assert qw.nonfinite_groups == 0
    Wf = inputs.bf16_bits_to_f32(W).astype(np.float64)
    Xf = inputs.bf16_bits_to_f32(X).astype(np.float64)
    q, s16, z16, _ = cal.gptq_quantize(Wf, Xf, sym=sym)
    P = oracle.pack_u4(q, sym)
    got_q = host_u32(qw.qweight)
    bad_rows = np.nonzero(np.any(got_q != P, axis=1))[0]
    assert bad_rows.size == 0, f"codes differ in rows {bad_rows[:10]}"
    assert np.array_equal(host_u16(qw.scales), s16), "fp16 scales differ"
    if not sym:
        assert np.array_equal(host_u16(qw.zeros), z16), "fp16 zeros differ"
    # the layout copy is the RTN layout of these buffers
    assert np.array_equal(qw.packed.cpu().numpy(), oracle.relayout(P, s16, z16, N, K, sym))
    return qw


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("N,K,T", [(64, 512, 768), (100, 384, 512), (33, 256, 300)])
def test_gptq_matches_the_oracle(N, K, T, sym):
    W = inputs.weights(N, K, 0.02, seed=N + K)
    X = inputs.correlated_calibration(T, K, seed=T + K)
    _compare_with_oracle(W, X, sym)


def test_gptq_matches_the_oracle_1024_inputs():
    """Eight groups, so the feedback crosses seven group boundaries and the
    Cholesky factorization spans 16 diagonal blocks."""
    W = inputs.weights(128, 1024, 0.015, seed=11)
    X = inputs.correlated_calibration(1024, 1024, seed=12)
    _compare_with_oracle(W, X, False)


def test_gptq_with_outlier_weights_and_channels():
    K = 512
    W = inputs.weights(96, K, 0.02, seed=21, outlier_frac=0.002)
    X = inputs.correlated_calibration(640, K, seed=22)
    Xf = inputs.bf16_bits_to_f32(X)
    Xf[:, inputs.outlier_channels(K, 0.01, seed=23)] *= 20.0
    _compare_with_oracle(W, inputs.to_bf16_bits(Xf), False)


def test_gptq_large_beats_rtn_and_is_deterministic():
    """4096 x 4096 (a Llama-7B attention projection) with 512 correlated
    calibration rows: the GPU codes decode to weights whose output error
    ||X W^T - X W_hat^T||^2 is well below plain RTN's, and two runs are
    bit-identical."""
    import torch
    N = K = 4096
    W = inputs.weights(N, K, 0.02, seed=31)
    X = inputs.correlated_calibration(512, K, seed=32)
    a = _gptq_gpu(W, X, False)
    b = _gptq_gpu(W, X, False)
    assert a.nonfinite_groups == 0
    assert torch.equal(a.qweight, b.qweight) and torch.equal(a.scales, b.scales)
    assert torch.equal(a.zeros, b.zeros)
    K_ = K
    W_gptq = oracle.dequant(host_u32(a.qweight), host_u16(a.scales), host_u16(a.zeros), K_)
    q, s, z, _ = oracle.quantize_bf16(W, None, sym=False)
    W_rtn = oracle.dequant(oracle.pack_u4(q, False), s, z, K_)
    Wf = inputs.bf16_bits_to_f32(W).astype(np.float64)
    Xf = inputs.bf16_bits_to_f32(X).astype(np.float64)
    rows = np.arange(0, N, 8)                           # a sample of output rows
    e_gptq = cal.output_error(Wf[rows], W_gptq[rows], Xf)
    e_rtn = cal.output_error(Wf[rows], W_rtn[rows], Xf)
    assert e_gptq < 0.8 * e_rtn, (e_gptq, e_rtn)


def test_gptq_status_reports_a_singular_hessian():
    """All-zero calibration inputs make H = 0 and its damping 0: the first
    Cholesky pivot is 0, reported in bit 1 of the status word."""
    W = inputs.weights(32, 256, 0.02, seed=41)
    X = np.zeros((64, 256), np.uint16)
    qw = _gptq_gpu(W, X, False)
    assert qw.nonfinite_groups & 2


def test_gptq_rejects_bad_arguments():
    import torch
    buf = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    need = abi.wq_gptq_workspace_bytes(8, 16, 256)
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    args = dict(W=buf, X=buf, T=8, N=16, K=256, group_size=128, symmetric=0, damp=0.01,
                qweight=buf, scales=buf, zeros=buf, workspace=ws, ws_bytes=need, d_status=None)
    assert abi.wq_gptq_quantize(**args) == abi.WQ_OK
    torch.cuda.synchronize()
    for k, v, st in (("K", 200, abi.WQ_ERR_UNSUPPORTED_SHAPE), ("T", 0, abi.WQ_ERR_UNSUPPORTED_SHAPE),
                     ("damp", -1.0, abi.WQ_ERR_INVALID_ARG), ("zeros", None, abi.WQ_ERR_INVALID_ARG),
                     ("ws_bytes", need - 1, abi.WQ_ERR_WORKSPACE_TOO_SMALL),
                     ("K", abi.WQ_GPTQ_MAX_K + 128, abi.WQ_ERR_UNSUPPORTED_SHAPE)):
        a = dict(args)
        a[k] = v
        assert abi.wq_gptq_quantize(**a) == st, k
