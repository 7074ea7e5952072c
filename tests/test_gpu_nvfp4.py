"""NVFP4 on the GPU against the oracle (oracle/nvfp4.py), "3.6 量化(Quantization)",
section 数值格式 (E2M1 elements, one E4M3 scale per 16, one fp32 scale per
tensor):

  * wq_nvfp4_quantize: codes, block scales and the tensor scale bit for bit;
  * wq_nvfp4_pack_layout: the scale layout of the tensor cores, from its
    definition;
  * wq_nvfp4_linear (both operands NVFP4, block-scaled FP4 tensor cores, fp32
    accumulation): within rel-L2 1e-3 and max-abs 1e-2 rms(y) of the oracle's
    fp64 product of the same dequantized operands."""
import numpy as np
import pytest

from oracle import nvfp4 as onv
import post_weight_quantization_wq_b200 as wq
from post_weight_quantization_wq_b200 import inputs
from gpu_util import check_close, dev_bf16, sample_rows

pytestmark = pytest.mark.gpu


def _gpu_quant(bits):
    codes, scales, S, st = wq.nvfp4_quantize_tensor(dev_bf16(bits))
    return (codes.cpu().numpy(), scales.cpu().numpy(), float(S[0].item()), int(st[0].item()))


def _oracle_quant(bits, S=None):
    c, sc, s = onv.nvfp4_quantize(inputs.bf16_bits_to_f32(bits), S=S)
    return onv.pack_e2m1(c), sc, s


def _sf_layout(sc, N, K):
    """The tensor cores' scale layout, from its definition (128-row tiles,
    512-byte blocks per 64 inputs, row 128 t + 32 m1 + m0 at m0*16 + m1*4)."""
    NBt = -(-N // 128)
    out = np.zeros((NBt, K // 64, 32, 4, 4), np.uint8)
    for r in range(N):
        t, m1, m0 = r // 128, (r // 32) % 4, r % 32
        out[t, :, m0, m1, :] = sc[r].reshape(K // 64, 4)
    return out.reshape(-1)


@pytest.mark.parametrize("N,K,sigma,outl", [(256, 1024, 0.02, 0.0), (100, 384, 0.015, 0.002),
                                            (1, 128, 1.0, 0.0), (333, 640, 3e-5, 0.01)])
def test_nvfp4_quantize_bit_exact(N, K, sigma, outl):
    W = inputs.weights(N, K, sigma, seed=N + K, outlier_frac=outl)
    codes, scales, S, st = _gpu_quant(W)
    rc, rs, rS = _oracle_quant(W)
    assert st == 0
    assert np.float32(S).view(np.uint32) == np.float32(rS).view(np.uint32)
    assert np.array_equal(scales, rs), "E4M3 block scales differ"
    assert np.array_equal(codes, rc), "E2M1 codes differ"


def test_nvfp4_quantize_activation_shape_and_zero_block():
    x = inputs.activations(3, 512, seed=4, channels=inputs.outlier_channels(512, 0.01, 5), mult=50.0)
    xf = inputs.bf16_bits_to_f32(x)
    xf[1, 32:48] = 0.0                       # an all-zero block: floor scale 2^-9, codes 0
    x = inputs.to_bf16_bits(xf)
    codes, scales, S, st = _gpu_quant(x)
    rc, rs, rS = _oracle_quant(x)
    assert np.array_equal(scales, rs) and np.array_equal(codes, rc)
    assert scales[1, 2] == 0x01


def test_nvfp4_pack_layout():
    N, K = 300, 768
    W = inputs.weights(N, K, 0.02, seed=9)
    qw = wq.nvfp4_quantize(dev_bf16(W))
    packed = qw.packed.cpu().numpy()
    codes = qw.codes.cpu().numpy()
    assert np.array_equal(packed[:N * K // 2], codes.reshape(-1))
    assert np.array_equal(packed[N * K // 2:], _sf_layout(qw.scales.cpu().numpy(), N, K))


def _linear_ref(x_bits, W_bits, rows=None):
    Wf = inputs.bf16_bits_to_f32(W_bits)
    S_w = onv.nvfp4_tensor_scale(Wf)
    if rows is not None:
        Wf = Wf[rows]
    wc, ws, _ = onv.nvfp4_quantize(Wf, S=S_w)
    xc, xs, xS = onv.nvfp4_quantize(inputs.bf16_bits_to_f32(x_bits))
    return onv.nvfp4_linear(xc, xs, xS, wc, ws, S_w)


@pytest.mark.parametrize("M", [1, 3, 16, 17, 64, 128])
@pytest.mark.parametrize("N,K", [(256, 1024), (200, 384), (130, 1408)])
def test_nvfp4_linear(N, K, M):
    W = inputs.weights(N, K, 0.02, seed=N * 3 + K)
    x = inputs.activations(M, K, seed=M + K)
    qw = wq.nvfp4_quantize(dev_bf16(W))
    y = wq.nvfp4_linear(dev_bf16(x), qw).cpu().numpy()
    check_close(y, _linear_ref(x, W), f"nvfp4 N={N} K={K} M={M}")


def test_nvfp4_linear_deterministic():
    import torch
    W = inputs.weights(512, 4096, 0.02, seed=1)
    x = dev_bf16(inputs.activations(4, 4096, seed=2))
    qw = wq.nvfp4_quantize(dev_bf16(W))
    assert torch.equal(wq.nvfp4_linear(x, qw), wq.nvfp4_linear(x, qw))


@pytest.mark.parametrize("M", [1, 16])
def test_nvfp4_linear_full_size(M):
    """The 8192 x 28672 down projection (K split across CTAs): sampled rows
    against the oracle (rows quantized with the whole tensor's scale)."""
    cid, li = 3, 3
    W = inputs.workload_weight(cid, li)
    x = inputs.workload_activations(cid, li, M)
    qw = wq.nvfp4_quantize(dev_bf16(W))
    y = wq.nvfp4_linear(dev_bf16(x), qw).cpu().numpy()
    rows = sample_rows(W.shape[0], n=96, seed=7)
    check_close(y[:, rows], _linear_ref(x, W, rows), f"nvfp4 8192x28672 M={M}")
