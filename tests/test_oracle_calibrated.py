"""Pins of the calibrated-quantizer oracle (GPTQ, AWQ alpha search).

Each check ties the oracle to something other than itself: the objective the
method minimizes written as an ordinary least-squares problem, special cases
that reduce to the pinned RTN routine, a matrix identity, the per-element
error bound the AWQ scaling argument rests on, and the improvements over RTN
the pages describe.
"""
import numpy as np
import pytest

import oracle
import oracle.calibrated as cal
from post_weight_quantization_wq_b200 import inputs

K = 256
G = 128


def _correlated_inputs(T, K, seed, mix=0.3):
    g = inputs.rng(seed)
    A = g.standard_normal((K, K)) * mix + np.eye(K)
    return g.standard_normal((T, K)) @ A


def _fp32_weights(N, K, seed, sigma=0.02):
    return (inputs.rng(seed).standard_normal((N, K)) * sigma).astype(np.float32).astype(np.float64)


def _rtn(W, sym):
    q, s16, z16, bad = oracle.quantize_f32(np.asarray(W, np.float32), G, 4, sym)
    assert bad == 0
    return q, s16, z16, oracle.dequant(oracle.pack_u4(q, sym), s16, z16, W.shape[1], G, sym)


# ------------------------------------------------------------------ GPTQ

@pytest.mark.parametrize("sym", [False, True])
def test_gptq_diagonal_hessian_is_rtn(sym):
    """Uncorrelated calibration features (X^T X diagonal) leave nothing to feed
    back: every off-diagonal entry of the remaining inverse is 0, so GPTQ
    reduces to per-group RTN (same codes, same scales and zeros)."""
    W = _fp32_weights(12, K, 11)
    d = 0.5 + inputs.rng(12).random(K)
    X = np.diag(d)                              # T = K rows, columns orthogonal
    q, s16, z16, W_cur = cal.gptq_quantize(W, X, G, sym)
    qr, sr, zr, Wr = _rtn(W, sym)
    np.testing.assert_array_equal(q, qr)
    np.testing.assert_array_equal(s16, sr)
    if not sym:
        np.testing.assert_array_equal(z16, zr)
    np.testing.assert_array_equal(W_cur, Wr)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("cols", [1, 2, 7, G, G + 3, K - 1])
def test_gptq_feedback_is_least_squares(sym, cols):
    """The objective ("3.6 量化" section GPTQ): after the first ``cols`` columns
    are fixed at their quantized values, the remaining columns must be the
    ordinary least-squares minimizer of ||X W^T - X W_cur^T||^2 over them.
    Undamped H; checked against numpy's lstsq on X itself, so a wrong sign,
    a transposed or stale inverse, or a wrong index fails it."""
    W = _fp32_weights(6, K, 21)
    X = _correlated_inputs(3 * K, K, 22)
    _, _, _, W_cur = cal.gptq_quantize(W, X, G, sym, damp=0.0, columns=cols)
    Q, F = slice(0, cols), slice(cols, K)
    rhs = X @ W.T - X[:, Q] @ W_cur[:, Q].T
    WF, *_ = np.linalg.lstsq(X[:, F], rhs, rcond=None)
    scale = np.max(np.abs(WF.T))
    np.testing.assert_allclose(W_cur[:, F], WF.T, rtol=0, atol=1e-9 * scale)


def test_gptq_error_never_decreases_with_columns():
    """Each fixed column adds a non-negative error term (the increase of a
    constrained quadratic minimum): the output error after c columns is
    non-decreasing in c, and 0 before the first column."""
    W = _fp32_weights(4, K, 31)
    X = _correlated_inputs(2 * K, K, 32)
    errs = []
    for c in (0, 1, 5, 64, 128, 129, 200, K):
        _, _, _, W_cur = cal.gptq_quantize(W, X, G, False, damp=0.0, columns=c)
        errs.append(cal.output_error(W, W_cur, X))
    assert errs[0] < 1e-20
    assert all(b >= a * (1 - 1e-9) for a, b in zip(errs, errs[1:])), errs


@pytest.mark.parametrize("sym", [False, True])
def test_gptq_beats_rtn_on_correlated_inputs(sym):
    """The error feedback lowers the layer's output error relative to RTN when
    the calibration features are correlated ("3.6 量化" section GPTQ: errors on
    correlated features can be absorbed by the others)."""
    W = _fp32_weights(16, K, 41)
    X = _correlated_inputs(2 * K, K, 42)
    _, _, _, W_g = cal.gptq_quantize(W, X, G, sym)
    *_, W_r = _rtn(W, sym)
    e_g, e_r = cal.output_error(W, W_g, X), cal.output_error(W, W_r, X)
    assert e_g < 0.7 * e_r, (e_g, e_r)


@pytest.mark.parametrize("sym", [False, True])
def test_gptq_output_format(sym):
    """Codes lie in the RTN code range, and the stored codes, scales and zeros
    dequantize exactly to the weights GPTQ settled on, so the packed result is
    a valid input of the W4A16 linear."""
    W = _fp32_weights(8, K, 51)
    X = _correlated_inputs(2 * K, K, 52)
    q, s16, z16, W_cur = cal.gptq_quantize(W, X, G, sym)
    lo, hi = (-7, 7) if sym else (0, 15)
    assert q.min() >= lo and q.max() <= hi
    Wd = oracle.dequant(oracle.pack_u4(q, sym), s16, z16, K, G, sym)
    np.testing.assert_array_equal(W_cur, Wd)


@pytest.mark.parametrize("sym", [False, True])
def test_gptq_weights_on_the_grid_are_a_fixed_point(sym):
    """Weights that already are RTN levels of their groups (with both extreme
    codes present in every group) give zero rounding error in every column:
    no feedback, and GPTQ returns the same codes for any calibration data."""
    g = inputs.rng(61)
    N = 8
    lo, hi = (-7, 7) if sym else (0, 15)
    q0 = g.integers(lo, hi + 1, size=(N, K)).astype(np.int32)
    q0[:, ::G] = lo
    q0[:, 1::G] = hi
    s16 = oracle.f32_to_f16_bits((0.001 + 0.01 * g.random((N, K // G))).astype(np.float32))
    z16 = None if sym else oracle.f32_to_f16_bits(np.full((N, K // G), 8.0, np.float32))
    W = oracle.dequant(oracle.pack_u4(q0, sym), s16, z16, K, G, sym)
    X = _correlated_inputs(2 * K, K, 62)
    q, s_out, z_out, W_cur = cal.gptq_quantize(W, X, G, sym)
    np.testing.assert_array_equal(q, q0)
    np.testing.assert_array_equal(s_out, s16)
    np.testing.assert_array_equal(W_cur, W)


def test_cholesky_rows_equal_the_sequential_inverse():
    """Reading G1: the rows of the upper Cholesky factor U of H^-1 (H^-1 = U^T U)
    carry the same update direction as the inverse of H restricted to the
    remaining columns: U[j, j:] / U[j, j] = inv(H[j:, j:])[0] / inv(H[j:, j:])[0, 0].
    This is the identity that lets a blocked implementation use one
    factorization instead of K inverses."""
    X = _correlated_inputs(2 * K, K, 71)
    H = cal.hessian(X, damp=0.01)
    U = np.linalg.cholesky(np.linalg.inv(H)).T
    for j in (0, 1, 63, 128, K - 2):
        r = np.linalg.inv(H[j:, j:])[0]
        np.testing.assert_allclose(U[j, j:] / U[j, j], r / r[0], rtol=0, atol=1e-9)


# ------------------------------------------------------------------ AWQ

def _awq_case(N=16, seed=5, mult=20.0, sym=False):
    ch = inputs.outlier_channels(K, 0.01, seed)
    Xb = inputs.activations(128, K, seed + 1, ch, mult)
    Wb = inputs.weights(N, K, 0.02, seed + 2)
    return Wb, Xb


@pytest.mark.parametrize("sym", [False, True])
def test_awq_alpha_zero_is_rtn(sym):
    """alpha = 0 gives s = 1 exactly, so the first grid point is plain RTN:
    its loss equals the loss of the RTN codes through the pinned linear."""
    Wb, Xb = _awq_case(sym=sym)
    res = cal.awq_search(Wb, Xb, G, sym)
    q, s16, z16, _ = oracle.quantize_bf16(Wb, None, G, sym)
    y = oracle.linear(Xb, oracle.pack_u4(q, sym), s16, z16, K, G, sym)
    W = oracle.bf16_to_f32(Wb).astype(np.float64)
    X = oracle.bf16_to_f32(Xb).astype(np.float64)
    assert res["losses"][0] == float(np.sum((X @ W.T - y) ** 2))


def test_awq_uniform_channel_magnitudes_give_a_flat_search():
    """When every channel has the same mean magnitude, s_X is constant, the
    normalized scale is 1 for every alpha, every grid point is RTN, and the
    first (alpha = 0) wins."""
    g = inputs.rng(81)
    X = np.where(g.random((128, K)) < 0.5, -1.0, 1.0).astype(np.float32)
    Xb = inputs.to_bf16_bits(X)
    Wb = inputs.weights(8, K, 0.02, 82)
    res = cal.awq_search(Wb, Xb, G, False)
    assert np.all(res["losses"] == res["losses"][0])
    assert res["alpha"] == 0.0
    assert np.all(res["s"] == np.float32(1.0))


@pytest.mark.parametrize("sym", [False, True])
def test_awq_effective_error_shrinks_by_s(sym):
    """The scaling argument ("3.6 量化" section AWQ): the rounding error of
    s_j w_j is at most half a step of its group, so the error of the weight
    the activations actually meet, quant(s_j w_j) / s_j, is at most
    step / (2 s_j).  A scale applied on the wrong axis or inverted fails it."""
    Wb, Xb = _awq_case(sym=sym)
    res = cal.awq_search(Wb, Xb, G, sym)
    s = res["s"].astype(np.float64)
    assert res["alpha"] > 0
    W = oracle.bf16_to_f32(Wb).astype(np.float64)
    W_eff = cal.effective_weights(Wb, res["s"], G, sym)
    _, s16, _, _ = oracle.quantize_bf16(Wb, res["s"], G, sym)
    step = np.repeat(oracle.f16_bits_to_f64(s16), G, axis=1)
    bound = (step / 2 * (1 + 2.0 ** -20) + np.abs(W * s) * 2.0 ** -23) / s[None, :]
    assert np.all(np.abs(W - W_eff) <= bound)


@pytest.mark.parametrize("sym", [False, True])
def test_awq_search_beats_rtn_on_outlier_channels(sym):
    """With 1 % of the input channels 20x larger than the rest, the search
    picks alpha > 0 and lowers the output error well below RTN's (the
    salient-channel observation of the AWQ sections)."""
    Wb, Xb = _awq_case(sym=sym)
    res = cal.awq_search(Wb, Xb, G, sym)
    assert 0 < res["alpha"] < 1
    assert res["losses"][res["i"]] < 0.6 * res["losses"][0]
    assert res["losses"][res["i"]] == res["losses"].min()


def test_awq_loss_matches_a_dense_recomputation():
    """The search's loss (through the C linear, which divides x by s) agrees
    with a dense numpy evaluation through the effective weights."""
    Wb, Xb = _awq_case(N=8, seed=9)
    res = cal.awq_search(Wb, Xb, G, False, n_grid=4)
    W = oracle.bf16_to_f32(Wb).astype(np.float64)
    X = oracle.bf16_to_f32(Xb).astype(np.float64)
    sx = np.maximum(np.mean(np.abs(X), axis=0), 1e-8)
    for i, a in enumerate(res["alphas"]):
        W_eff = cal.effective_weights(Wb, cal.awq_scale(sx, float(a)), G, False)
        dense = float(np.sum((X @ (W - W_eff).T) ** 2))
        assert abs(res["losses"][i] - dense) <= 1e-9 * dense


def test_awq_scale_follows_channel_magnitude():
    """Reading A1: for alpha > 0 the scale grows with the channel's mean
    magnitude (outlier channels get the largest s), and its geometric mean is
    1 up to the fp32 rounding of each s_j."""
    Wb, Xb = _awq_case()
    X = oracle.bf16_to_f32(Xb).astype(np.float64)
    sx = np.mean(np.abs(X), axis=0)
    for a in (0.25, 0.5, 1.0):
        s = cal.awq_scale(sx, a).astype(np.float64)
        order = np.argsort(sx)
        assert np.all(np.diff(s[order]) >= 0)
        assert abs(np.mean(np.log(s))) < 2.0 ** -22
        ch = inputs.outlier_channels(K, 0.01, 5)
        assert s[ch].min() > np.delete(s, ch).max()
