"""CPU oracle for NVFP4 block-scaled 4-bit floating point: E2M1 elements in
blocks of 16 along the input dimension, one FP8 E4M3 scale per block and one
fp32 scale per tensor; plus the linear that consumes it.

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only ``tests/``, the smoke
check and the benchmark's CPU legs may import it, and it imports nothing from
the CUDA library.  Both number formats are decoded and encoded here from
their bit layouts, value by value (slow, plain Python / numpy).

Sources (page title, then section / table):
  [3.6]  "3.6 量化(Quantization)", section 数值格式 (its format table: FP8 E4M3
         is 1 sign / 4 exponent / 3 mantissa bits with largest value 448; FP4
         E2M1 is 1 / 2 / 1 bits with magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6;
         NVFP4 is 16 E2M1 elements sharing one E4M3 scale plus one fp32 scale
         per tensor; MXFP4 is 32 elements with a power-of-two E8M0 scale),
         section 粒度 (per-block scales of 16 or 32 elements) and section
         实例演算 (4 + 8/16 = 4.5 bits per element for NVFP4).
  [Pano] "大模型量化全景解析", section 3 "Scale、Zero Point、Group Size" (block-wise
         scales fitted to the hardware tile, for FP8/FP4/MX formats).

Readings where the pages leave a step open:
  F1  E2M1 (bias 1, no infinities or NaN): encoding rounds to the nearest
      magnitude, ties to the even code, and saturates at 6; the sign is kept
      (a negative value that rounds to 0 is -0).
  F2  E4M3 (bias 7, no infinities, S.1111.111 is NaN, largest 448): encoding
      rounds to nearest even and saturates at 448.
  F3  Tensor scale S = max(amax(W), 1e-8) / (6 * 448) in fp32 (each step of
      F3-F5 is one fp32 operation, correctly rounded), so the largest
      block scale lands on the largest E4M3 value.
  F4  Block scale: d = amax_b / fl(6 S) in fp32, stored as E4M3(d); a block
      scale that rounds to 0 becomes the smallest E4M3 subnormal 2^-9.
  F5  Element code: E2M1(w / fl(s_b S)) with the quotient rounded to fp32.
  F6  Dequantization w_hat = E2M1(q) * E4M3(s_b) * S, exact in fp64.
  F7  Finite input only: a NaN or infinity in W is refused (ValueError).
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 16
E4M3_MAX = 448.0
E2M1_MAX = 6.0


# --------------------------------------------------------------- E2M1 (FP4)

def e2m1_decode(code: int) -> float:
    """Value of a 4-bit E2M1 code: bit 3 sign, bits 2..1 exponent (bias 1),
    bit 0 mantissa; exponent 0 is subnormal (0.5 * m)."""
    sign = -1.0 if code & 8 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    mag = 0.5 * m if e == 0 else (1.0 + 0.5 * m) * 2.0 ** (e - 1)
    return sign * mag


_E2M1_MAGS = [e2m1_decode(c) for c in range(8)]          # ascending


def e2m1_encode(v: float) -> int:
    """Reading F1: nearest magnitude, ties to the even code, saturate at 6."""
    if not math.isfinite(v):
        raise ValueError("e2m1_encode: non-finite value")
    a = abs(v)
    sign = 8 if math.copysign(1.0, v) < 0 else 0
    if a >= E2M1_MAX:
        return sign | 7
    best = 0
    for c in range(1, 8):
        d_new, d_best = abs(a - _E2M1_MAGS[c]), abs(a - _E2M1_MAGS[best])
        if d_new < d_best or (d_new == d_best and c % 2 == 0):
            best = c
    return sign | best


# --------------------------------------------------------------- E4M3 (FP8)

def e4m3_decode(code: int) -> float:
    """Value of an 8-bit E4M3 code: bit 7 sign, bits 6..3 exponent (bias 7),
    bits 2..0 mantissa; exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is
    NaN; there are no infinities."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 15
    m = code & 7
    if e == 15 and m == 7:
        return float("nan")
    mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return sign * mag


_E4M3_POS = [(e4m3_decode(c), c) for c in range(0x7F)]   # finite, non-negative, ascending


def e4m3_encode(v: float) -> int:
    """Reading F2: round to nearest, ties to the even code, saturate at 448."""
    if math.isnan(v):
        return 0x7F
    a = abs(v)
    sign = 0x80 if math.copysign(1.0, v) < 0 else 0
    if a >= E4M3_MAX:
        return sign | 0x7E
    lo, hi = 0, len(_E4M3_POS) - 1            # binary search for the bracketing pair
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if _E4M3_POS[mid][0] <= a:
            lo = mid
        else:
            hi = mid
    (vl, cl), (vh, ch) = _E4M3_POS[lo], _E4M3_POS[hi]
    if a - vl < vh - a:
        return sign | cl
    if a - vl > vh - a:
        return sign | ch
    return sign | (cl if cl % 2 == 0 else ch)


# --------------------------------------------------------------- NVFP4

def _f32(v) -> float:
    return float(np.float32(v))


def nvfp4_tensor_scale(W) -> float:
    """Reading F3: S = max(amax(W), 1e-8) / (6 * 448), rounded to fp32."""
    W = np.asarray(W, np.float32)
    amax = float(np.max(np.abs(W))) if W.size else 0.0
    return _f32(max(amax, _f32(1e-8)) / (E2M1_MAX * E4M3_MAX))


def nvfp4_quantize(W, block: int = BLOCK, S=None):
    """NVFP4 quantization of W [rows][cols] (blocks of ``block`` consecutive
    columns).  Returns (codes uint8 [rows][cols], one E2M1 code per byte;
    block scales uint8 [rows][cols/block], E4M3 codes; tensor scale S as an
    fp32 value).  ``S``: the tensor scale to use (default: the one of W, reading
    F3), so rows of a larger tensor can be quantized on their own."""
    W = np.asarray(W, np.float32)
    rows, cols = W.shape
    if cols % block:
        raise ValueError("nvfp4_quantize: cols must be a multiple of the block")
    if not np.all(np.isfinite(W)):
        raise ValueError("nvfp4_quantize: non-finite weights")           # F7
    if S is None:
        S = nvfp4_tensor_scale(W)                                         # F3
    S6 = _f32(E2M1_MAX * S)
    codes = np.zeros((rows, cols), np.uint8)
    scales = np.zeros((rows, cols // block), np.uint8)
    for r in range(rows):
        for b in range(cols // block):
            blk = W[r, b * block:(b + 1) * block]
            amax_b = float(np.max(np.abs(blk)))
            sb = e4m3_encode(_f32(amax_b / S6))                           # F4
            if sb == 0:
                sb = 0x01
            scales[r, b] = sb
            eff = _f32(e4m3_decode(sb) * S)
            for i in range(block):
                codes[r, b * block + i] = e2m1_encode(_f32(float(blk[i]) / eff))   # F5
    return codes, scales, S


def nvfp4_dequant(codes, scales, S: float, block: int = BLOCK) -> np.ndarray:
    """w_hat = E2M1(q) * E4M3(s_b) * S in fp64 (reading F6)."""
    codes = np.asarray(codes, np.uint8)
    scales = np.asarray(scales, np.uint8)
    e2 = np.array([e2m1_decode(c) for c in range(16)])
    e4 = np.array([e4m3_decode(c) for c in range(256)])
    return e2[codes] * np.repeat(e4[scales], block, axis=1) * float(S)


def pack_e2m1(codes) -> np.ndarray:
    """Two codes per byte, element 2i in the low nibble (the byte order of
    the packed FP4 operand)."""
    c = np.asarray(codes, np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def nvfp4_linear(x_codes, x_scales, x_S, w_codes, w_scales, w_S, block: int = BLOCK):
    """y = dequant(x) dequant(W)^T in fp64, both operands NVFP4 (the FP4
    tensor-core form: activations quantized the same way as the weights)."""
    return nvfp4_dequant(x_codes, x_scales, x_S, block) @ \
        nvfp4_dequant(w_codes, w_scales, w_S, block).T
