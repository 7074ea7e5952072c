"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print, closed forms, an independent conversion routine, exact rational
arithmetic, or brute force over every quantization level.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = [float(v) for v in vals]
    return out


def _f16(h):
    return float(oracle.f16_bits_to_f64(np.array([h], np.uint16))[0])


# --------------------------------------------------------------- P1 / P2

@pytest.mark.parametrize("form", ["sym", "asym"])
def test_worked_example_int4(form):
    """P1/P2: the page's hand-worked 8-value INT4 example ("3.6 量化" 实例演算)."""
    g = _read_golden("worked_example_int4.txt")
    w = np.array(g["values"], np.float32)[None, :]
    sym = form == "sym"
    q, s16, z16, bad = oracle.quantize_f32(w, group=8, bits=4, sym=sym)
    assert bad == 0
    s = _f16(s16[0, 0])
    assert abs(s - g[f"{form}.s"][0]) < 6e-5
    assert q[0].tolist() == [int(v) for v in g[f"{form}.q"]]
    z = 0.0 if sym else _f16(z16[0, 0])
    if not sym:
        assert z == g["asym.z"][0]
    xhat = s * (q[0].astype(np.float64) - z)
    np.testing.assert_allclose(xhat, g[f"{form}.xhat"], atol=6e-4)
    mse = float(np.mean((w[0].astype(np.float64) - xhat) ** 2))
    assert abs(mse - g[f"{form}.mse"][0]) <= 0.006e-3


# --------------------------------------------------------------- P3

def test_outlier_step_zeroes_the_rest():
    """P3: one 100 among values of size ~1 gives a 4-bit step of ~100/7 and
    every other value rounds to 0 ("3.6 量化" section 直觉)."""
    g = _read_golden("self_test_answers.txt")
    r = np.random.default_rng(3)
    w = r.uniform(-2.0, 2.0, size=128).astype(np.float32)
    w[37] = g["outlier.value"][0]
    q, s16, _, bad = oracle.quantize_f32(w[None, :], group=128, bits=4, sym=True)
    assert bad == 0
    s = _f16(s16[0, 0])
    assert abs(s - g["outlier.step"][0]) < 0.01
    others = np.delete(q[0], 37)
    assert np.all(others == 0)
    assert q[0, 37] == 7


# --------------------------------------------------------------- P4

def test_int8_self_test_answer():
    """P4: symmetric INT8 with max|x| = 2.54 has step 0.02 and 1.0 maps to 50
    ("3.6 量化" section 自测); the oracle takes any bit width."""
    g = _read_golden("self_test_answers.txt")
    w = np.zeros((1, 16), np.float32)
    w[0, 0] = g["int8_sym.max"][0]
    w[0, 1] = 1.0
    q, s16, _, _ = oracle.quantize_f32(w, group=16, bits=8, sym=True)
    assert abs(_f16(s16[0, 0]) - g["int8_sym.step"][0]) < 1e-5
    assert q[0, 1] == int(g["int8_sym.q_of_1"][0])
    assert q[0, 0] == 127


# --------------------------------------------------------------- P5

@pytest.mark.parametrize("sym,key", [(True, "g128_f16scale.bits"),
                                     (False, "g128_f16scale_f16zero.bits")])
def test_effective_bits_from_buffers(sym, key):
    """P5: bits per weight counted from the buffers the oracle emits equal the
    pages' 4 + 16/128 (scale) and 4 + 32/128 (scale + zero)."""
    g = _read_golden("self_test_answers.txt")
    r = np.random.default_rng(5)
    N, K = 64, 1024
    w = (r.standard_normal((N, K)) * 0.02).astype(np.float32)
    q, s16, z16, _ = oracle.quantize_f32(w, group=128, bits=4, sym=sym)
    P = oracle.pack_u4(q, sym)
    nbytes = P.nbytes + s16.nbytes + (0 if sym else z16.nbytes)
    assert 8 * nbytes / (N * K) == g[key][0]
    # the page's G=64 variant with an fp16 scale and an INT4 zero, by formula
    assert 4 + (16 + 4) / 64 == g["g64_f16scale_int4zero.bits"][0]


# --------------------------------------------------------------- P6

@pytest.mark.parametrize("sym", [True, False])
def test_error_bound_half_step(sym):
    """P6: |w - x_hat| <= s/2 for every element not clipped ("3.6 量化" section
    对称与非对称量化), plus the fp32 division's rounding of w/s."""
    r = np.random.default_rng(6 + sym)
    N, K = 96, 1024
    w = (r.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[r.random((N, K)) < 0.002] *= 25.0                 # outliers
    w[5, 128:256] = 0.0                                 # all-zero group
    w[6, 0:128] = np.abs(w[6, 0:128]) + 0.5             # zero not in range
    q, s16, z16, bad = oracle.quantize_f32(w, group=128, bits=4, sym=sym)
    assert bad == 0
    s = oracle.f16_bits_to_f64(s16).repeat(128, axis=1)
    z = 0.0 if sym else oracle.f16_bits_to_f64(z16).repeat(128, axis=1)
    xhat = s * (q - z)
    err = np.abs(w.astype(np.float64) - xhat)
    lo, hi = (-7, 7) if sym else (0, 15)
    inner = (q > lo) & (q < hi)
    t = np.abs(w / s)
    assert np.all(err[inner] <= s[inner] * (0.5 + t[inner] * 2.0 ** -23))
    # elements at the clamp ends are within half a step unless truly clipped
    ends = ~inner
    clipped = err[ends] > s[ends] * (0.5 + t[ends] * 2.0 ** -23)
    # a clipped element must lie beyond the last level on its side
    qe, xe, we = q[ends][clipped], xhat[ends][clipped], w[ends][clipped]
    assert np.all(np.where(qe == hi, we > xe, we < xe))


# --------------------------------------------------------------- P7

def test_group_vs_tensor_error_ratio():
    """P7: on rows with scales spread over logspace(-2, 0), per-group-128 INT4
    error is about a third of per-tensor error ("3.6 量化" section 代码)."""
    r = np.random.default_rng(0)
    W = (r.standard_normal((256, 1024)) * np.logspace(-2, 0, 256)[:, None]).astype(np.float32)

    def rel_err(group, rows, cols):
        w = W.reshape(rows, cols)
        q, s16, _, _ = oracle.quantize_f32(w, group=group, bits=4, sym=True)
        s = oracle.f16_bits_to_f64(s16).repeat(group, axis=1)
        wh = (s * q).reshape(W.shape)
        return np.linalg.norm(W - wh) / np.linalg.norm(W)

    e_tensor = rel_err(256 * 1024, 1, 256 * 1024)
    e_channel = rel_err(1024, 256, 1024)
    e_group = rel_err(128, 256, 1024)
    assert e_tensor > e_channel > e_group
    assert 0.25 <= e_group / e_tensor <= 0.45


# --------------------------------------------------------------- P8

def _brute_force_check(w_row, q_row, s_bits, z_bits, sym):
    """Each code must be a nearest level among all 16; ties go to even RTN."""
    s = Fraction(_f16(s_bits))
    z = Fraction(0) if sym else Fraction(_f16(z_bits))
    levels = range(-7, 8) if sym else range(0, 16)
    for w, q in zip(w_row, q_row):
        W = Fraction(float(w))
        d = {c: abs(W - s * (c - z)) for c in levels}
        best = min(d.values())
        winners = [c for c in levels if d[c] == best]
        t = W / s
        near_tie = abs(abs(t - math.floor(t)) - Fraction(1, 2)) <= abs(t) * Fraction(1, 2 ** 23)
        if near_tie and not len(winners) > 1:
            # fp32 division may land on either side of an almost-tie
            ordered = sorted(levels, key=lambda c: d[c])
            assert q in ordered[:2]
            continue
        assert q in winners, (float(w), q, winners)
        if len(winners) > 1:
            # exact tie: round half to even on w/s
            n = int(q - z)
            assert n % 2 == 0


@pytest.mark.parametrize("sym", [True, False])
def test_brute_force_nearest_level(sym):
    """P8: on tiny groups, every RTN code is the nearest of all 16 levels
    (ties, planted exactly, resolved to even)."""
    r = np.random.default_rng(8 + sym)
    rows = []
    for _ in range(300):
        G = int(r.integers(2, 5))
        vals = r.choice(np.arange(-8, 9) / 4.0, size=G) * float(r.choice([1, 0.03, 7.5]))
        rows.append((G, vals.astype(np.float32)))
    # exact half-steps: max 0.875 with s = 0.125 (sym) / range 1.875 (asym)
    for k in range(-7, 7):
        if sym:
            rows.append((3, np.array([0.875, 0.125 * (k + 0.5), -0.3], np.float32)))
        else:
            rows.append((3, np.array([-0.875, 1.0, 0.125 * (k + 0.5)], np.float32)))
    for G, vals in rows:
        q, s16, z16, bad = oracle.quantize_f32(vals[None, :], group=G, bits=4, sym=sym)
        if bad:
            # a constant group whose fp16 zero point overflows (asymmetric only)
            assert not sym and np.all(vals == vals[0]) and vals[0] != 0
            continue
        _brute_force_check(vals, q[0], s16[0, 0], None if sym else z16[0, 0], sym)


# --------------------------------------------------------------- P9

def test_awq_fold_identity():
    """P9: (X diag(s)^-1)(diag(s) W) = X W ("3.6 量化" section SmoothQuant, the
    identity AWQ's fold relies on; "后训练量化" section AWQ steps 3 and 5)."""
    r = np.random.default_rng(9)
    K = 1024
    W = (r.standard_normal((8, K)) * 0.02).astype(np.float32)
    x = r.standard_normal(K).astype(np.float32)
    s = np.exp(r.uniform(-1.5, 1.5, K)).astype(np.float32)
    Wf = oracle.awq_fold_weight(W, s)
    lhs = (x.astype(np.float64) / s.astype(np.float64)) @ Wf.astype(np.float64).T
    rhs = x.astype(np.float64) @ W.astype(np.float64).T
    np.testing.assert_allclose(lhs, rhs, rtol=2e-6, atol=1e-9)
    wrong = (x.astype(np.float64) * s) @ Wf.astype(np.float64).T
    assert not np.allclose(wrong, rhs, rtol=1e-2)


def test_awq_linear_divides_activations():
    """The oracle's AWQ linear applies x / s per input channel: with power-of-
    two s, x = x~ * s gives exactly the plain linear of x~."""
    r = np.random.default_rng(10)
    N, K = 16, 512
    from post_weight_quantization_wq_b200 import inputs
    W = inputs.weights(N, K, 0.02, seed=11)
    s = (2.0 ** r.integers(-2, 3, K)).astype(np.float32)
    q, s16, z16, bad = oracle.quantize_bf16(W, s, sym=False)
    assert bad == 0
    P = oracle.pack_u4(q, False)
    xt = inputs.activations(2, K, seed=12)
    x = inputs.to_bf16_bits(inputs.bf16_bits_to_f32(xt) * s)   # exact: powers of two
    y_awq = oracle.linear(x, P, s16, z16, K, sym=False, awq_s=s)
    y_plain = oracle.linear(xt, P, s16, z16, K, sym=False)
    assert np.array_equal(y_awq, y_plain)


# --------------------------------------------------------------- P10

def test_f16_conversion_special_values():
    """P10 (part): IEEE binary16 RNE at the edges, against numpy's converter."""
    vals = np.array([0.0, -0.0, 1.0, 65504.0, 65519.99, 65520.0, 1e6, -1e6,
                     2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.0000001, 3 * 2.0 ** -26,
                     2.0 ** -14, 2.0 ** -14 - 2.0 ** -25, 0.1, 1.0009765625 + 2 ** -11,
                     float("inf"), -float("inf")], np.float32)
    got = oracle.f32_to_f16_bits(vals)
    ref = vals.astype(np.float16).view(np.uint16)
    assert got.tolist() == ref.tolist()
    assert (oracle.f32_to_f16_bits(np.array([np.nan], np.float32))[0] & 0x7C00) == 0x7C00


def test_f16_conversion_random_vs_numpy():
    r = np.random.default_rng(10)
    bits = r.integers(0, 2 ** 32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    assert np.array_equal(oracle.f32_to_f16_bits(f), f.astype(np.float16).view(np.uint16))


def test_f16_conversion_exhaustive():
    """P10: against the host compiler's _Float16 cast, every fp32 bit pattern
    whose biased exponent lies in [98, 145] (all of binary16's rounding:
    half-quantum underflow at 2^-25 up to overflow at 65520, both signs),
    and a stride through all 2^32 patterns (the rest map to +-0, +-inf, NaN)."""
    for sign in (0, 1 << 31):
        lo = sign | (98 << 23)
        hi = sign | (146 << 23)
        assert oracle.f16_selfcheck(lo, hi) == 0
    assert oracle.f16_selfcheck(0, 2 ** 32, 997) == 0


def test_round_half_even():
    cases = {0.5: 0.0, 1.5: 2.0, 2.5: 2.0, -0.5: -0.0, -1.5: -2.0, -2.5: -2.0,
             0.49999997: 0.0, 2.5000002: 3.0, 7.0: 7.0, -7.4: -7.0, 8388607.5: 8388608.0}
    for v, e in cases.items():
        assert oracle.round_half_even(v) == e
    r = np.random.default_rng(1)
    for v in (r.standard_normal(20000) * 20).astype(np.float32):
        assert oracle.round_half_even(float(v)) == float(np.rint(v))


# --------------------------------------------------------------- P11

def test_linear_fp64_against_exact_sum():
    """P11: the oracle's fp64 accumulation against math.fsum of the exact
    products (x is bf16, x_hat an fp16 times a small integer: every product is
    exact in fp64), on the single-linear workload."""
    from post_weight_quantization_wq_b200 import inputs
    W, x, _ = inputs.workload_inputs(1, 0, 1)
    q, s16, z16, bad = oracle.quantize_bf16(W, None, sym=False)
    assert bad == 0
    P = oracle.pack_u4(q, False)
    rows = np.arange(0, 256, 7)
    y = oracle.linear(x, P, s16, z16, 1024, sym=False, rows=rows)[0]
    xh = oracle.dequant(P, s16, z16, 1024, sym=False)
    xf = inputs.bf16_bits_to_f32(x)[0].astype(np.float64)
    for i, n in enumerate(rows):
        terms = xf * xh[n]
        exact = math.fsum(terms.tolist())
        assert abs(y[i] - exact) <= 1024 * 2.0 ** -52 * np.sum(np.abs(terms))


# --------------------------------------------------------------- packing

def test_pack_nibble_order():
    """Canonical packing: element k = 8j + i of a row in bits [4i, 4i+4) of
    word j; symmetric codes stored as q + 8."""
    q = np.arange(16, dtype=np.int32)[None, :] % 16
    P = oracle.pack_u4(q, sym=False)
    assert P[0].tolist() == [0x76543210, 0xFEDCBA98]
    qs = np.array([[-7, -6, -5, -4, -3, -2, -1, 0]], np.int32)
    assert oracle.pack_u4(qs, sym=True)[0].tolist() == [0x87654321]
    r = np.random.default_rng(2)
    qa = r.integers(0, 16, size=(5, 256)).astype(np.int32)
    assert np.array_equal(oracle.unpack_u4(oracle.pack_u4(qa, False), 256, False), qa)


# --------------------------------------------------------------- degenerate groups

def test_degenerate_groups():
    w = np.zeros((1, 512), np.float32)
    w[0, 128:256] = 0.25                    # constant positive group
    w[0, 256:384] = np.linspace(0.5, 0.51, 128, dtype=np.float32)
    w[0, 400] = np.inf
    q, s16, z16, bad = oracle.quantize_f32(w, 128, 4, sym=False)
    # all-zero group: tiny scale 2^-24, zero +0, codes 0
    assert s16[0, 0] == 0x0001 and z16[0, 0] == 0x0000 and np.all(q[0, :128] == 0)
    # constant positive group: the zero point exceeds fp16 -> non-finite
    assert s16[0, 1] == 0x7E00 and z16[0, 1] == 0x7E00
    # zero outside [0, 15] is stored exactly and codes stay in range
    z = _f16(z16[0, 2])
    assert z < 0 and z == int(z) and q[0, 256:384].min() >= 0 and q[0, 256:384].max() <= 15
    assert s16[0, 3] == 0x7E00
    assert bad == 2
    qs, ss, _, bads = oracle.quantize_f32(w, 128, 4, sym=True)
    assert bads == 1 and ss[0, 3] == 0x7E00 and np.all(qs[0, 384:] == -8)
    assert ss[0, 0] == 0x0001 and np.all(qs[0, :128] == 0)
