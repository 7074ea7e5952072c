"""CPU oracle for the two calibrated quantizers that build on per-group RTN:
the GPTQ column-sequential quantizer and the AWQ search over the scale
exponent alpha.

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only ``tests/``, the smoke
check and the benchmark's CPU legs may import it.  It imports nothing from the
CUDA library.  Floating point is fp64 (the pages fix no precision for either
method); the group parameters, the codes' stored format, the packing, the
dequantization and the AWQ-folded RTN are the pinned C routines of this
package, so both quantizers emit exactly the format the W4A16 linear reads.

Sources (page title, then section / equation):
  [3.6]  "3.6 量化(Quantization)", section GPTQ (objective min ||WX - W_hat X||^2
         over the calibration inputs; after quantizing input column j with
         error e_j = w_j - quant(w_j), W[:, F] -= e_j / [H^-1]_jj * [H^-1]_{j,F}
         over the not yet quantized columns F, H = 2 X X^T), section AWQ
         (s = s_X^alpha, s_X the mean activation magnitude per input channel,
         grid search of alpha in [0, 1] per layer minimizing the output error
         on the calibration data; y = sum_j quant(s_j w_j) x_j / s_j).
  [Inf]  "推理优化中“用精度换性能“的核心技术：量化", section 四.2 (columns in
         natural order, H from the calibration inputs, per-column error
         feedback into the remaining columns) and 四.4 (one scale per group of
         128 columns).
  [Pano] "大模型量化全景解析", section 六.2 "GPTQ：用二阶信息做 one-shot 权重量化"
         (its parameter table: damp_percent, a damping term added to the
         Hessian for numerical stability; sym; group_size).

Readings where the pages leave a step open:
  G1  [H^-1] in the update is the inverse of H restricted to the columns not yet
      quantized (the exact sequential OBS form; the fast Cholesky form computes
      the same rows).  The inference-optimization page's "invert once, reuse
      the full inverse" is read as a simplification, not the method.
  G2  Damping: H + damp * mean(diag H) * I with damp = 0.01 by default
      (damp_percent is named, its default is not given).
  G3  The scale (and zero) of a group come from the RTN rules applied to the
      group's 128 current weights at the moment its first column is quantized
      (after the feedback of all earlier columns), rounded to fp32 first, as
      the RTN path does; the codes of every column of the group use them.
  G4  Codes: q = clamp(rint(w / s16) + z16), rint = round half to even, the
      division in fp64 on the fp64 working weights.
  A1  s_X_j = mean_t |X_tj| over the calibration rows, floored at 1e-8; for
      each alpha, s = s_X^alpha divided by its geometric mean (so the product
      of the s_j is 1), rounded to fp32 (the format the quantizer takes).
  A2  The grid is alpha = i / n_grid, i = 0..n_grid, n_grid = 20; the loss is
      ||X W^T - (X diag(s)^-1) dequant(Q(W diag(s)))^T||_F^2 in fp64; the
      smallest alpha among equal minima wins.
"""
from __future__ import annotations

import numpy as np

from . import (GROUP, bf16_to_f32, dequant, f16_bits_to_f64, linear, pack_u4,
               quantize_bf16, quantize_f32)


def _code_range(sym: bool, bits: int = 4):
    if sym:
        qmax = (1 << (bits - 1)) - 1
        return -qmax, qmax
    return 0, (1 << bits) - 1


def hessian(X, damp: float = 0.01) -> np.ndarray:
    """H = 2 X^T X (X: calibration inputs [T][K], one row per token), plus the
    damping term of reading G2."""
    X = np.asarray(X, np.float64)
    H = 2.0 * (X.T @ X)
    if damp:
        H = H + damp * float(np.mean(np.diag(H))) * np.eye(H.shape[0])
    return H


def gptq_quantize(W, X, group: int = GROUP, sym: bool = False, damp: float = 0.01,
                  columns: int | None = None):
    """GPTQ ([3.6] GPTQ, [Inf] 四.2): quantize the input columns of W [N][K]
    one at a time in natural order, feeding each column's rounding error
    back into the columns not yet quantized through the inverse Hessian of
    the calibration inputs X [T][K].

    ``columns`` stops after that many columns (None = all K); the columns
    after it then hold the compensated, still unquantized weights.

    Returns (q int32 [N][K] signed codes, s16 uint16 [N][K/group], z16 uint16
    [N][K/group] or None, W_cur fp64 [N][K]): q, s16 and z16 are in the RTN
    format (codes of columns past ``columns`` are 0); W_cur holds the
    dequantized value of every quantized column and the compensated weights
    of the rest."""
    W = np.array(W, dtype=np.float64)
    N, K = W.shape
    assert K % group == 0
    H = hessian(X, damp)
    assert H.shape == (K, K)
    stop = K if columns is None else int(columns)
    qlo, qhi = _code_range(sym)
    q = np.zeros((N, K), np.int32)
    s16 = np.zeros((N, K // group), np.uint16)
    z16 = None if sym else np.zeros((N, K // group), np.uint16)
    s = z = None
    for j in range(stop):
        g = j // group
        if j % group == 0:                       # G3: parameters of group g, now
            block = W[:, j:j + group].astype(np.float32)
            _, sg, zg, bad = quantize_f32(block, group, 4, sym)
            if bad:
                raise ValueError(f"gptq: non-finite weights in group {g}")
            s16[:, g] = sg[:, 0]
            s = f16_bits_to_f64(sg[:, 0])
            if sym:
                z = np.zeros(N)
            else:
                z16[:, g] = zg[:, 0]
                z = f16_bits_to_f64(zg[:, 0])
        col = W[:, j]
        qj = np.clip(np.rint(col / s) + z, qlo, qhi)   # G4
        w_hat = s * (qj - z)
        e = col - w_hat
        Hinv = np.linalg.inv(H[j:, j:])                  # G1: remaining columns only
        W[:, j + 1:] -= np.outer(e / Hinv[0, 0], Hinv[0, 1:])
        W[:, j] = w_hat
        q[:, j] = qj.astype(np.int32)
    return q, s16, z16, W


def output_error(W_ref, W_hat, X) -> float:
    """||X W_ref^T - X W_hat^T||_F^2 in fp64 (the objective of [3.6] GPTQ)."""
    D = np.asarray(W_ref, np.float64) - np.asarray(W_hat, np.float64)
    return float(np.sum((np.asarray(X, np.float64) @ D.T) ** 2))


def awq_scale(sx, alpha: float) -> np.ndarray:
    """s = s_X^alpha over its geometric mean, in fp32 (reading A1)."""
    m = np.asarray(sx, np.float64) ** alpha
    m = m / np.exp(np.mean(np.log(m)))
    return m.astype(np.float32)


def awq_search(W_bits, X_bits, group: int = GROUP, sym: bool = False, n_grid: int = 20):
    """AWQ scale search ([3.6] AWQ): for alpha on the grid of reading A2,
    fold s = s_X^alpha into the weights, quantize them with per-group RTN,
    and measure the output error of the layer on the calibration inputs with
    the activations divided by s.  W_bits: bf16 bit patterns [N][K];
    X_bits: bf16 calibration inputs [T][K].

    Returns a dict: alphas [n_grid+1], losses [n_grid+1] (fp64), best index
    ``i``, ``alpha`` and its scale ``s`` (fp32 [K])."""
    W = bf16_to_f32(W_bits).astype(np.float64)
    X = bf16_to_f32(X_bits).astype(np.float64)
    N, K = W.shape
    sx = np.maximum(np.mean(np.abs(X), axis=0), 1e-8)
    y_ref = X @ W.T
    alphas = np.arange(n_grid + 1, dtype=np.float64) / n_grid
    losses = np.empty(n_grid + 1)
    scales = []
    for i, a in enumerate(alphas):
        s = awq_scale(sx, float(a))
        q, s16, z16, bad = quantize_bf16(W_bits, awq_s=s, group=group, sym=sym)
        if bad:
            raise ValueError(f"awq_search: {bad} non-finite groups at alpha={a}")
        y = linear(X_bits, pack_u4(q, sym), s16, z16, K, group, sym, awq_s=s)
        losses[i] = float(np.sum((y_ref - y) ** 2))
        scales.append(s)
    best = int(np.argmin(losses))                        # first of equal minima
    return {"alphas": alphas, "losses": losses, "i": best,
            "alpha": float(alphas[best]), "s": scales[best]}


def effective_weights(W_bits, s, group: int = GROUP, sym: bool = False) -> np.ndarray:
    """dequant(Q(W diag(s))) diag(s)^-1 in fp64: the weights the AWQ linear
    applies to the unscaled activations."""
    q, s16, z16, bad = quantize_bf16(W_bits, awq_s=s, group=group, sym=sym)
    if bad:
        raise ValueError("effective_weights: non-finite groups")
    K = q.shape[1]
    Wd = dequant(pack_u4(q, sym), s16, z16, K, group, sym)
    return Wd / np.asarray(s, np.float32).astype(np.float64)[None, :]
