"""Seeded synthetic inputs shared by the tests, the oracle checks and the bench.

This module holds only random-number recipes and the workload table; it does
none of the quantization or linear arithmetic, and it imports neither the CUDA
library nor the oracle.  Every array is produced from NumPy's PCG64 stream in
fp32 and rounded to bf16 (round to nearest even, done by torch's dtype
conversion) where a bf16 tensor is wanted.  bf16 tensors are returned as
uint16 bit patterns so both sides can take them without conversion.

Workloads follow the decode-linear shapes the quantization pages discuss
(Llama-2-7B / 70B, "推理优化中“用精度换性能“的核心技术：量化" section 一,
"3.6 量化(Quantization)" section 实例演算); the distributions (N(0, 0.02),
N(0, 0.015) weights, 0.1 % +-20 sigma weight outliers, 1 % activation
outlier channels) are the synthetic stand-in for real checkpoints and
activations, which this library never loads.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

GROUP = 128


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (round to nearest even) as uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def weights(N: int, K: int, sigma: float, seed: int, outlier_frac: float = 0.0,
            outlier_sigmas: float = 20.0) -> np.ndarray:
    """bf16 W [N][K] ~ N(0, sigma^2); with ``outlier_frac`` > 0, exactly
    round(outlier_frac*N*K) positions (uniform, without replacement) are set
    to +-outlier_sigmas*sigma with a random sign."""
    g = rng(seed)
    w = g.standard_normal((N, K), dtype=np.float32)
    w *= np.float32(sigma)
    n_out = int(round(outlier_frac * N * K))
    if n_out:
        pos = g.choice(N * K, size=n_out, replace=False)
        sign = np.where(g.random(n_out) < 0.5, -1.0, 1.0).astype(np.float32)
        w.reshape(-1)[pos] = sign * np.float32(outlier_sigmas * sigma)
    return to_bf16_bits(w)


def outlier_channels(K: int, frac: float, seed: int) -> np.ndarray:
    """A fixed set of ceil(frac*K) input channels (sorted indices)."""
    n = int(math.ceil(frac * K))
    return np.sort(rng(seed).choice(K, size=n, replace=False))


def activations(M: int, K: int, seed: int, channels: np.ndarray | None = None,
                mult: float = 1.0) -> np.ndarray:
    """bf16 x [M][K] ~ N(0, 1); the given input channels are multiplied by
    ``mult`` (the same channels for every row)."""
    x = rng(seed).standard_normal((M, K), dtype=np.float32)
    if channels is not None and len(channels):
        x[:, channels] *= np.float32(mult)
    return to_bf16_bits(x)


def awq_scale_from_calibration(X: np.ndarray, alpha: float = 0.5) -> np.ndarray:
    """The per-input-channel scale of the AWQ workload: s_j = (mean_t |X_tj|)^alpha,
    divided by its geometric mean so that prod_j s_j = 1.  X: fp32 [T][K].
    This is the workload's fixed recipe for s (no search); the quantizer and
    the linear only consume s."""
    m = np.mean(np.abs(X.astype(np.float64)), axis=0) ** alpha
    m = m / math.exp(float(np.mean(np.log(m))))
    return m.astype(np.float32)


def correlated_calibration(T: int, K: int, seed: int, mix: float = 1.0) -> np.ndarray:
    """bf16 calibration inputs X [T][K] with correlated features:
    X = Z (I + mix * A / sqrt(K)), Z and A standard normal (fp32), so every
    feature mixes in about mix^2 of the others' variance whatever K is (the
    case the GPTQ error feedback is for; independent features would make it
    plain RTN)."""
    g = rng(seed)
    Z = g.standard_normal((T, K), dtype=np.float32)
    A = g.standard_normal((K, K), dtype=np.float32)
    A *= np.float32(mix / math.sqrt(K))
    A[np.diag_indices(K)] += np.float32(1.0)
    return to_bf16_bits(Z @ A)


@dataclass
class Linear:
    name: str
    N: int
    K: int
    sigma: float
    seed: int
    outlier_frac: float = 0.0


@dataclass
class Workload:
    cid: int
    title: str
    linears: list
    Ms: list
    sym: bool
    act_outlier_frac: float = 0.0
    act_outlier_mult: float = 1.0
    awq: bool = False
    calib_rows: int = 0
    calib_outlier_mult: float = 1.0
    notes: str = ""
    extra: dict = field(default_factory=dict)


def _lin(cid, i, name, N, K, sigma, **kw):
    seed = 0 if cid == 1 else 1000 * cid + i
    return Linear(name, N, K, sigma, seed, **kw)


WORKLOADS = {
    1: Workload(1, "single linear 256x1024, asymmetric, M=1",
                [_lin(1, 0, "w", 256, 1024, 0.02)], [1], sym=False),
    2: Workload(2, "Llama-7B-shaped decode linears, symmetric, 0.1% +-20 sigma outliers, M=1",
                [_lin(2, 0, "attn", 4096, 4096, 0.02, outlier_frac=0.001),
                 _lin(2, 1, "up", 11008, 4096, 0.02, outlier_frac=0.001),
                 _lin(2, 2, "down", 4096, 11008, 0.02, outlier_frac=0.001)],
                [1], sym=True),
    3: Workload(3, "Llama-70B-shaped decode linears, asymmetric, M in {1,2,4,8}",
                [_lin(3, 0, "qo", 8192, 8192, 0.015),
                 _lin(3, 1, "kv", 1024, 8192, 0.015),
                 _lin(3, 2, "gate_up", 28672, 8192, 0.015),
                 _lin(3, 3, "down", 8192, 28672, 0.015)],
                [1, 2, 4, 8], sym=False),
    4: Workload(4, "batched-decode skinny GEMM, asymmetric, 1% activation channels x30",
                [_lin(4, 0, "gate_up", 28672, 8192, 0.015),
                 _lin(4, 1, "down", 8192, 28672, 0.015)],
                [16, 32, 64], sym=False, act_outlier_frac=0.01, act_outlier_mult=30.0),
    5: Workload(5, "Llama-70B GQA decoder layer, AWQ fold, asymmetric, M in {1,4}",
                [_lin(5, 0, "q", 8192, 8192, 0.015),
                 _lin(5, 1, "k", 1024, 8192, 0.015),
                 _lin(5, 2, "v", 1024, 8192, 0.015),
                 _lin(5, 3, "o", 8192, 8192, 0.015),
                 _lin(5, 4, "gate", 28672, 8192, 0.015),
                 _lin(5, 5, "up", 28672, 8192, 0.015),
                 _lin(5, 6, "down", 8192, 28672, 0.015)],
                [1, 4], sym=False, act_outlier_frac=0.01, act_outlier_mult=50.0,
                awq=True, calib_rows=128, calib_outlier_mult=50.0),
}


def act_seed(cid: int, lin_index: int, M: int) -> int:
    return 1000 * cid + 100 + 10 * lin_index + M % 10 + 7 * (M // 10)


def calib_seed(cid: int, K: int) -> int:
    return 1000 * cid + 200 + (K // 1024)


def outlier_seed(cid: int, K: int) -> int:
    return 1000 * cid + 300 + (K // 1024)


def workload_weight(cid: int, lin_index: int) -> np.ndarray:
    lin = WORKLOADS[cid].linears[lin_index]
    return weights(lin.N, lin.K, lin.sigma, lin.seed, lin.outlier_frac)


def _channels(cid: int, K: int):
    wl = WORKLOADS[cid]
    if not wl.act_outlier_frac:
        return None
    return outlier_channels(K, wl.act_outlier_frac, outlier_seed(cid, K))


def workload_activations(cid: int, lin_index: int, M: int) -> np.ndarray:
    wl = WORKLOADS[cid]
    K = wl.linears[lin_index].K
    return activations(M, K, act_seed(cid, lin_index, M), _channels(cid, K), wl.act_outlier_mult)


def workload_awq_scale(cid: int, lin_index: int):
    """The AWQ scale of the workload's linear, or None.  The calibration rows
    and the runtime rows share one distribution and one set of outlier
    channels per input size K."""
    wl = WORKLOADS[cid]
    if not wl.awq:
        return None
    K = wl.linears[lin_index].K
    X = bf16_bits_to_f32(activations(wl.calib_rows, K, calib_seed(cid, K), _channels(cid, K),
                                     wl.calib_outlier_mult))
    return awq_scale_from_calibration(X)


def workload_inputs(cid: int, lin_index: int, M: int):
    """(W bits [N][K], x bits [M][K], awq_s fp32 [K] or None) for one linear of
    a workload."""
    return (workload_weight(cid, lin_index), workload_activations(cid, lin_index, M),
            workload_awq_scale(cid, lin_index))
