"""Pins of the NVFP4 oracle (E2M1 elements, E4M3 block scales, fp32 tensor
scale).

Each check ties the oracle to something other than itself: the values the
chapter-3.6 format table prints, PyTorch's own float8_e4m3fn conversion (an
independent library routine), brute force over every representable level,
exact round trips of values built from codes, and the block-isolation and
storage claims of the pages.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle.nvfp4 as nv
from post_weight_quantization_wq_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fp_formats.txt")


def _golden():
    out = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, *v = line.split()
                out[k] = [float(t) for t in v]
    return out


# ------------------------------------------------------------------ E2M1

def test_e2m1_values_are_the_pages_magnitudes():
    """The eight non-negative codes decode to the magnitudes the format table
    prints, and the negative codes to their negatives."""
    mags = _golden()["e2m1_magnitudes"]
    assert [nv.e2m1_decode(c) for c in range(8)] == mags
    for c in range(8):
        assert nv.e2m1_decode(c | 8) == -mags[c] or (c == 0 and nv.e2m1_decode(8) == 0.0)
    assert math.copysign(1.0, nv.e2m1_decode(8)) == -1.0


def test_e2m1_encode_is_nearest_level_ties_even():
    """Brute force over a dense grid (every tie point included): the code is
    a nearest magnitude; at a tie it is the even code; above 6 it saturates."""
    mags = _golden()["e2m1_magnitudes"]
    for a in np.arange(0, 8.0001, 1.0 / 64):
        a = float(a)
        c = nv.e2m1_encode(a)
        assert c < 8
        d = [abs(a - m) for m in mags]
        best = min(d)
        if a >= 6:
            assert c == 7
            continue
        assert abs(d[c] - best) == 0.0, (a, c)
        ties = [i for i in range(8) if d[i] == best]
        if len(ties) > 1:
            assert c in ties and c % 2 == 0, (a, c, ties)
        assert nv.e2m1_encode(-a) == (c | 8)


# ------------------------------------------------------------------ E4M3

def test_e4m3_decode_matches_torch_for_every_code():
    """All 256 codes against torch.float8_e4m3fn (NaN at S.1111.111 only), and
    the largest finite value is the table's 448."""
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float()
    for c in range(256):
        mine, theirs = nv.e4m3_decode(c), float(ref[c])
        if math.isnan(theirs):
            assert math.isnan(mine), c
        else:
            assert mine == theirs and math.copysign(1, mine) == math.copysign(1, theirs), c
    finite = [nv.e4m3_decode(c) for c in range(256) if not math.isnan(nv.e4m3_decode(c))]
    assert max(finite) == _golden()["e4m3_max"][0]


def test_e4m3_encode_matches_torch_rne_in_range():
    """Round to nearest even agrees with torch's fp32 -> float8_e4m3fn cast for
    every value up to 464 (the rounding midpoint above 448): all codes, every
    midpoint between neighbours, subnormals, random values.  Above that the
    oracle saturates at 448 (reading F2) where torch's cast gives NaN."""
    vals = [nv.e4m3_decode(c) for c in range(0x7F)]
    mids = [(a + b) / 2 for a, b in zip(vals, vals[1:])]
    rnd = list(inputs.rng(3).random(2000) * 464.0) + list(inputs.rng(4).random(500) * 2.0 ** -6)
    test = np.array(vals + mids + rnd + [464.0], np.float32)
    test = np.concatenate([test, -test])
    ref = torch.from_numpy(test).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for v, r in zip(test, ref):
        assert nv.e4m3_encode(float(v)) == int(r), (float(v), nv.e4m3_encode(float(v)), int(r))
    assert nv.e4m3_encode(500.0) == 0x7E and nv.e4m3_encode(1e30) == 0x7E


# ------------------------------------------------------------------ NVFP4

def _levels_weights(rows, cols, seed):
    """Weights built from codes: every block holds a +-6 element, block scales
    are E4M3 values and the largest block scale is 448, with S a power of
    two, so every step of the quantizer is exact."""
    g = inputs.rng(seed)
    S = 2.0 ** -12
    codes = g.integers(0, 16, size=(rows, cols)).astype(np.uint8)
    codes[:, ::16] = np.where(g.random((rows, cols // 16)) < 0.5, 7, 15)
    scales = g.integers(0x08, 0x7F, size=(rows, cols // 16)).astype(np.uint8)   # normal E4M3
    scales[0, 0] = 0x7E                                                          # 448
    W = nv.nvfp4_dequant(codes, scales, S)
    assert np.all(W.astype(np.float32) == W)
    return W, codes, scales, S


def test_nvfp4_round_trip_of_representable_weights():
    """Weights that are NVFP4 values (one +-6 per block, largest block scale
    448, power-of-two tensor scale) quantize back to the same codes, block
    scales and tensor scale."""
    W, codes, scales, S = _levels_weights(6, 64, 11)
    c2, s2, S2 = nv.nvfp4_quantize(W)
    assert S2 == S
    np.testing.assert_array_equal(s2, scales)
    # -0 and +0 are the same value; compare decoded values, then the rest exactly
    np.testing.assert_array_equal(nv.nvfp4_dequant(c2, s2, S2), W)
    nz = (codes & 7) != 0
    np.testing.assert_array_equal(c2[nz], codes[nz])


def test_nvfp4_error_within_half_a_local_step():
    """Every element lies within half the local E2M1 spacing (0.5 below 2, 1
    below 4, 2 up to 6) of its level, in units of the block's effective scale;
    the block maximum maps to at most 6 * (1 + 2^-4) (E4M3 rounding of the
    block scale), so nothing saturates by more than that."""
    W = inputs.bf16_bits_to_f32(inputs.weights(8, 256, 0.02, 21, outlier_frac=0.01)).astype(np.float64)
    codes, scales, S = nv.nvfp4_quantize(W)
    e4 = np.array([nv.e4m3_decode(c) for c in range(256)])
    eff = np.repeat(e4[scales], 16, axis=1) * S
    u = W / eff
    lvl = nv.nvfp4_dequant(codes, scales, S) / eff
    a = np.abs(u)
    half = np.where(a < 2, 0.25, np.where(a < 4, 0.5, 1.0))
    inside = a <= 6
    assert np.all(np.abs(u - lvl)[inside] <= half[inside] * (1 + 2.0 ** -20))
    assert np.all(a <= 6 * (1 + 2.0 ** -4) * (1 + 2.0 ** -20))


def test_nvfp4_outlier_stays_in_its_block():
    """The format table's point about block scales: an outlier stretches only
    its own block.  Raising one element (not the tensor maximum) changes the
    codes and scale of that block and of no other."""
    W = inputs.bf16_bits_to_f32(inputs.weights(4, 128, 0.02, 31)).astype(np.float64)
    W[0, 0] = 1.0                                       # the tensor maximum, fixed
    c1, s1, S1 = nv.nvfp4_quantize(W)
    W2 = W.copy()
    W2[2, 37] = 0.5                                     # block (2, 2)
    c2, s2, S2 = nv.nvfp4_quantize(W2)
    assert S1 == S2
    changed = np.argwhere(s1 != s2)
    assert changed.tolist() == [[2, 2]]
    diff_blocks = {(r, k // 16) for r, k in np.argwhere(c1 != c2)}
    assert diff_blocks == {(2, 2)}


def test_nvfp4_storage_is_4_5_bits_per_element():
    """4-bit codes packed two per byte plus one 8-bit scale per 16 elements:
    4.5 bits per element (section 实例演算), the fp32 tensor scale aside."""
    W = inputs.bf16_bits_to_f32(inputs.weights(8, 512, 0.02, 41)).astype(np.float64)
    codes, scales, S = nv.nvfp4_quantize(W)
    packed = nv.pack_e2m1(codes)
    bits = 8 * (packed.nbytes + scales.nbytes) / W.size
    assert bits == _golden()["nvfp4_bits_per_element"][0]
    assert W.shape[1] // scales.shape[1] == int(_golden()["nvfp4_block"][0])
    lo = packed & 0xF
    np.testing.assert_array_equal(lo, codes[:, 0::2])
    np.testing.assert_array_equal(packed >> 4, codes[:, 1::2])


def test_nvfp4_zero_and_tiny_blocks():
    """An all-zero tensor and an all-zero block quantize to zero codes with
    the floor block scale 2^-9 (reading F4) and dequantize to zero."""
    Z = np.zeros((2, 32))
    c, s, S = nv.nvfp4_quantize(Z)
    assert np.all((c & 7) == 0) and np.all(s == 0x01)
    assert np.all(nv.nvfp4_dequant(c, s, S) == 0)
    W = np.zeros((1, 32))
    W[0, 0] = 1.0
    c, s, S = nv.nvfp4_quantize(W)
    assert s[0, 0] == 0x7E and s[0, 1] == 0x01 and np.all((c[0, 16:] & 7) == 0)
    assert nv.e4m3_decode(0x01) == 2.0 ** -9


def test_nvfp4_refuses_non_finite():
    W = np.zeros((1, 16))
    W[0, 3] = np.inf
    with pytest.raises(ValueError):
        nv.nvfp4_quantize(W)


def test_nvfp4_linear_is_the_product_of_dequantized_operands():
    """The W4A4 linear equals an exact rational evaluation of
    sum_k x_hat_k w_hat_k on a small case (every dequantized value is a dyadic
    rational, so fp64 products are exact and only the sums round)."""
    from fractions import Fraction
    W = inputs.bf16_bits_to_f32(inputs.weights(3, 32, 0.02, 51)).astype(np.float64)
    X = inputs.bf16_bits_to_f32(inputs.activations(2, 32, 52)).astype(np.float64)
    wc, ws, wS = nv.nvfp4_quantize(W)
    xc, xs, xS = nv.nvfp4_quantize(X)
    y = nv.nvfp4_linear(xc, xs, xS, wc, ws, wS)
    Wd, Xd = nv.nvfp4_dequant(wc, ws, wS), nv.nvfp4_dequant(xc, xs, xS)
    for m in range(2):
        for n in range(3):
            exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(Xd[m], Wd[n]))
            assert abs(Fraction(float(y[m, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 40) + \
                Fraction(1, 2 ** 200)
