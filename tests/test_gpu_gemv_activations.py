"""The GEMV's integer paths (the tensor-core decode kernel, M = 2..8, and the
CUDA-core kernel, M <= 4; each case run on the default choice and with the
CUDA cores forced) on activations that stress their per-chunk 16-bit fixed
point: each 64-input chunk of a row of x is
rounded to x_i = rn(x * 2^e) with the chunk's largest |x| in [2^14, 2^15), so
small values next to large ones in one chunk lose low bits.  The pages
multiply the dequantized weights with the 16-bit activations themselves
("3.6 量化(Quantization)", section 仅权重 vs 权重 + 激活), which the fp64 oracle
does exactly; the kernel's rounding must stay inside the parity tolerance
(rel-L2 <= 1e-3, max-abs <= 1e-2 * rms(y)) on:

  * the outlier-channel recipes of the batched-decode and AWQ workloads
    (1 % of input channels x30 and x50), without the AWQ factor;
  * one element x1000 inside a chunk;
  * chunks whose magnitudes differ by 2^+-40;
  * all-zero chunks and an all-zero row;
  * tiny normal and subnormal bf16 activations (with weights large enough
    that y stays a normal fp32 number);
  * and a NaN or an infinity in x, which makes every output of that row
    non-finite (NaN) while the other rows stay exact."""
import numpy as np
import pytest

import oracle
import post_weight_quantization_wq_b200 as wq
from post_weight_quantization_wq_b200 import inputs
from gpu_util import check_close, dev_bf16, quantize_and_check, sample_rows

# every case on both decode kernels (tensor-core and CUDA-core integer paths)
pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("decode_kernel")]

N_SMALL, K_SMALL = 512, 4096


def _run(W, x, sym, what):
    qw, P, s, z = quantize_and_check(W, None, sym)
    y = wq.linear(dev_bf16(x), qw, path="gemv").cpu().numpy()
    yref = oracle.linear(x, P, s, z, W.shape[1], sym=sym)
    check_close(y, yref, what)
    return y, yref


@pytest.fixture(scope="module")
def w_small():
    return inputs.weights(N_SMALL, K_SMALL, 0.015, seed=5)


@pytest.mark.parametrize("mult", [30.0, 50.0])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 6, 8])
@pytest.mark.parametrize("sym", [False, True])
def test_outlier_channels(w_small, M, mult, sym):
    ch = inputs.outlier_channels(K_SMALL, 0.01, seed=6)
    x = inputs.activations(M, K_SMALL, seed=7 + M, channels=ch, mult=mult)
    _run(w_small, x, sym, f"outlier channels x{mult} M={M}")


@pytest.mark.parametrize("M", [1, 4])
def test_one_large_element_in_a_chunk(w_small, M):
    xf = np.random.default_rng(8).standard_normal((M, K_SMALL)).astype(np.float32)
    xf[:, 100] *= 1000.0
    xf[M - 1, 2000] *= 1000.0
    _run(w_small, inputs.to_bf16_bits(xf), False, f"x1000 element M={M}")


@pytest.mark.parametrize("M", [1, 3, 4])
def test_chunk_magnitudes_far_apart(w_small, M):
    xf = np.random.default_rng(9).standard_normal((M, K_SMALL)).astype(np.float32)
    sc = 2.0 ** np.random.default_rng(10 + M).choice([-40, 0, 40], size=(M, K_SMALL // 64))
    xf *= np.repeat(sc, 64, axis=1).astype(np.float32)
    _run(w_small, inputs.to_bf16_bits(xf), False, f"chunk scales 2^+-40 M={M}")


def test_zero_chunks_and_zero_row(w_small):
    M = 4
    xf = np.random.default_rng(11).standard_normal((M, K_SMALL)).astype(np.float32)
    xf[:, 0:64] = 0.0
    xf[:, 640:1280] = 0.0
    xf[2, :] = 0.0
    xf[3, 64:4096] = 0.0
    xf[3, 70] = 1.0
    x = inputs.to_bf16_bits(xf)
    y, yref = _run(w_small, x, False, "zero chunks")
    assert np.all(y[2] == 0.0) and np.all(yref[2] == 0.0)


@pytest.mark.parametrize("scale,what", [(1e-36, "tiny normal"), (1e-39, "subnormal")])
@pytest.mark.parametrize("M", [1, 4])
def test_tiny_and_subnormal_activations(M, scale, what):
    # weights around 1e4 (fp16 scales near 1e3) keep y a normal fp32 number
    W = inputs.weights(N_SMALL, K_SMALL, 1e4, seed=12)
    xf = (np.random.default_rng(13 + M).standard_normal((M, K_SMALL)) * scale).astype(np.float32)
    x = inputs.to_bf16_bits(xf)
    if what == "subnormal":
        assert np.all((x & 0x7F80) == 0)             # every element is a bf16 subnormal (or 0)
    _run(W, x, False, f"{what} x M={M}")


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf])
@pytest.mark.parametrize("M", [1, 4])
def test_non_finite_activation_gives_non_finite_row(w_small, M, bad):
    qw, P, s, z = quantize_and_check(w_small, None, False)
    xf = np.random.default_rng(15).standard_normal((M, K_SMALL)).astype(np.float32)
    r = M - 1
    xf[r, 1234] = bad
    x = inputs.to_bf16_bits(xf)
    y = wq.linear(dev_bf16(x), qw, path="gemv").cpu().numpy()
    yref = oracle.linear(x, P, s, z, K_SMALL, sym=False)
    # the row holding the bad value: every output non-finite on both sides
    # (the oracle gives +-inf or NaN, the kernel NaN, as its reading states)
    assert np.all(~np.isfinite(yref[r]))
    assert np.all(np.isnan(y[r]))
    keep = np.arange(M) != r
    if keep.any():
        check_close(y[keep], yref[keep], "rows without the bad value")


def test_full_size_down_projection_outlier_channels():
    """8192 x 28672 at M = 1 with the AWQ workload's activation recipe (1 %
    of channels x50), quantized without the AWQ factor, so the integer path
    sees the outlier channels; sampled rows against the oracle."""
    cid, li = 5, 6
    lin = inputs.WORKLOADS[cid].linears[li]
    W = inputs.workload_weight(cid, li)
    qw, P, s, z = quantize_and_check(W, None, False)
    del W
    rows = sample_rows(lin.N, seed=56)
    for M in (1, 4):
        x = inputs.workload_activations(cid, li, M)
        y = wq.linear(dev_bf16(x), qw, path="gemv").cpu().numpy()
        yref = oracle.linear(x, P, s, z, lin.K, sym=False, rows=rows)
        check_close(y[:, rows], yref, f"8192x28672 outlier channels x50 M={M}")
