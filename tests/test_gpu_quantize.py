"""GPU quantize + pack + relayout against the CPU oracle: bit-exact codes,
packed words, fp16 scales and zeros, kernel-layout bytes and non-finite
group counts."""
import numpy as np
import pytest

from post_weight_quantization_wq_b200 import inputs
from gpu_util import quantize_and_check

pytestmark = pytest.mark.gpu


def _special_weights(N, K, seed):
    """Normal weights with planted degenerate groups (see the oracle's rules)."""
    r = np.random.default_rng(seed)
    w = (r.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[0, 0:128] = 0.0                                        # all-zero group
    if K >= 256:
        w[0, 128:256] = 0.3                                  # constant positive group
    if N > 1:
        w[1, 0:128] = np.abs(w[1, 0:128]) + 0.5              # zero not in range
    if N > 2:
        w[2, 0:128] = 1e-7 * r.standard_normal(128)          # fp16 subnormal scale
    if N > 3:
        w[3, 0:128] *= 1e6                                   # scale overflows fp16
    if N > 4:
        w[4, 5] = np.inf
    if N > 5:
        w[5, 7] = np.nan
    if N > 6:
        # exact half steps: max 0.875 (s = 0.125), values at (k + 1/2) * 0.125
        w[6, 0:128] = 0.0
        w[6, 0] = 0.875
        w[6, 1:15] = 0.125 * (np.arange(-7, 7) + 0.5)
        w[6, 16] = -0.875
    return inputs.to_bf16_bits(w)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("N,K", [(1, 128), (7, 256), (200, 640), (256, 1024), (130, 1408),
                                 (300, 11008)])
def test_quantize_small_shapes_with_special_groups(N, K, sym):
    W = _special_weights(N, K, seed=N * 7 + K)
    quantize_and_check(W, None, sym)


@pytest.mark.parametrize("sym", [False, True])
def test_quantize_with_awq_scale(sym):
    N, K = 192, 1536
    W = inputs.weights(N, K, 0.015, seed=77)
    r = np.random.default_rng(78)
    s = np.exp(r.uniform(-2, 2, K)).astype(np.float32)
    quantize_and_check(W, s, sym)


def test_quantize_awq_overflow_is_nonfinite():
    N, K = 4, 256
    W = inputs.weights(N, K, 0.02, seed=5)
    s = np.ones(K, np.float32)
    s[3] = 3e38                                               # w * s overflows fp32
    qw, *_ = quantize_and_check(W, s, False)
    assert qw.nonfinite_groups >= 1


def test_quantize_outlier_weights_config2_shape():
    W = inputs.weights(512, 4096, 0.02, seed=2000, outlier_frac=0.001)
    quantize_and_check(W, None, True)


def _near_tie_inputs(sym):
    """W = 1.0 everywhere and an AWQ scale that places each w' = fp32(1 * s_k)
    exactly where its quotient by the group's fp16 scale lies just beside a
    half-integer (by 0 to 1e-4 relative, both sides) or on it: the quantizer
    must round every one exactly as an IEEE division would."""
    r = np.random.default_rng(12)
    K, N = 128 * 8, 4
    s_awq = np.empty(K, np.float32)
    for g in range(K // 128):
        amax = np.float32(r.uniform(0.3, 3.0))
        if sym:
            s16 = np.float16(amax / np.float32(7.0))
            lo, hi = -7, 6
        else:
            s16 = np.float16((amax - (-amax)) / np.float32(15.0))
            lo, hi = -8, 6
        vals = [amax, -amax]
        rel = [0.0, 1e-9, 1e-8, 1e-7, 5e-7, 1e-6, 3e-6, 1e-5, 1e-4]
        while len(vals) < 128:
            m = r.integers(lo, hi + 1)
            d = rel[r.integers(len(rel))] * (1 if r.random() < 0.5 else -1)
            v = np.float32(np.float64(s16) * (m + 0.5) * (1.0 + d))
            if abs(v) < amax:
                vals.append(v)
        s_awq[g * 128:(g + 1) * 128] = np.array(vals, np.float32)
    W = inputs.to_bf16_bits(np.ones((N, K), np.float32))
    return W, s_awq


@pytest.mark.parametrize("sym", [True, False])
def test_quantize_near_ties(sym):
    W, s_awq = _near_tie_inputs(sym)
    quantize_and_check(W, s_awq, sym)
