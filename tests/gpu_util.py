"""Helpers shared by the GPU parity tests: host<->device marshalling of the
seeded inputs and the tolerance check.  The expected values always come from
the CPU oracle; nothing here computes the method."""
import numpy as np

import oracle
from post_weight_quantization_wq_b200 import inputs

REL_L2_TOL = 1e-3          # relative L2 error of y against the fp64 oracle
MAX_ABS_TOL = 1e-2         # max |error| <= MAX_ABS_TOL * rms(y)


def dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).cuda().view(
        torch.bfloat16)


def dev_f32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def host_u32(t):
    return t.cpu().numpy().view(np.uint32)


def host_u16(t):
    return t.contiguous().cpu().numpy().view(np.uint16)


def check_close(y, yref, what=""):
    y = np.asarray(y, np.float64)
    yref = np.asarray(yref, np.float64)
    assert y.shape == yref.shape, (y.shape, yref.shape)
    err = y - yref
    rel = np.linalg.norm(err) / max(np.linalg.norm(yref), 1e-300)
    rms = np.sqrt(np.mean(yref ** 2))
    mx = np.max(np.abs(err)) if err.size else 0.0
    assert rel <= REL_L2_TOL, f"{what} rel-L2 {rel:.3e}"
    assert mx <= MAX_ABS_TOL * rms, f"{what} max-abs {mx:.3e} vs rms {rms:.3e}"
    return rel, mx / rms


def oracle_quantize(W, awq, sym):
    q, s, z, bad = oracle.quantize_bf16(W, awq, sym=sym)
    P = oracle.pack_u4(q, sym)
    del q
    return P, s, z, bad


def sample_rows(N, n=384, seed=0):
    """Output rows to check at full size: random ones plus tile edges."""
    r = np.random.default_rng(seed)
    edges = [0, 1, 15, 16, 127, 128, N // 2, N - 129, N - 128, N - 2, N - 1]
    rows = np.concatenate([r.choice(N, size=min(n, N), replace=False),
                           np.array([e for e in edges if 0 <= e < N])])
    return np.unique(rows).astype(np.int64)


def quantize_and_check(W, awq, sym):
    """Quantize on the GPU, compare every integer output with the oracle
    bit for bit, and return (QuantizedWeight, P, s, z)."""
    import post_weight_quantization_wq_b200 as wq
    N, K = W.shape
    qw = wq.quantize(dev_bf16(W), None if awq is None else dev_f32(awq), symmetric=sym)
    P, s, z, bad = oracle_quantize(W, awq, sym)
    assert qw.nonfinite_groups == bad
    assert np.array_equal(host_u32(qw.qweight), P), "packed codes differ"
    assert np.array_equal(host_u16(qw.scales), s), "fp16 scales differ"
    if not sym:
        assert np.array_equal(host_u16(qw.zeros), z), "fp16 zeros differ"
    ref_layout = oracle.relayout(P, s, z, N, K, sym)
    assert np.array_equal(qw.packed.cpu().numpy(), ref_layout), "kernel layout differs"
    return qw, P, s, z
