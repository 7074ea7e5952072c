"""CPU oracle for per-group RTN 4-bit weight quantization and the W4A16 linear.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never imports it, and it imports nothing from the library: the two share no
code.  The arithmetic lives in plain C (``wq_oracle.c``, built with gcc, no
fused multiply-add); this module only marshals numpy arrays through ctypes.

What each function follows is stated beside it and in ``wq_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SOURCES = ("wq_oracle.c", "f16_selfcheck.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_wq.so")
_lock = threading.Lock()
_lib = None

GROUP = 128


def build_oracle(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle_wq.so`` (gcc, -O2, no FMA
    contraction, IEEE semantics).  Rebuilds when a source is newer."""
    srcs = [os.path.join(_HERE, s) for s in _SOURCES]
    if not force and os.path.exists(_LIB_PATH):
        lib_m = os.path.getmtime(_LIB_PATH)
        if all(os.path.getmtime(s) <= lib_m for s in srcs):
            return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-ffp-contract=off",
           "-fno-fast-math", "-fopenmp", "-o", tmp] + srcs + ["-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build_oracle())
        P = ctypes.c_void_p
        I = ctypes.c_int64
        C = ctypes.c_int
        sig = {
            "or_bf16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
            "or_f16_to_f64": (ctypes.c_double, [ctypes.c_uint16]),
            "or_f32_to_f16": (ctypes.c_uint16, [ctypes.c_float]),
            "or_f32_to_f16_array": (None, [P, P, I]),
            "or_f16_to_f64_array": (None, [P, P, I]),
            "or_round_half_even": (ctypes.c_float, [ctypes.c_float]),
            "or_quantize_f32": (I, [P, I, I, I, C, C, P, P, P]),
            "or_awq_fold_weight": (None, [P, P, I, I, P]),
            "or_quantize_bf16": (I, [P, P, I, I, I, C, P, P, P]),
            "or_pack_u4": (None, [P, I, I, C, P]),
            "or_unpack_u4": (None, [P, I, I, C, P]),
            "or_dequant": (None, [P, P, P, I, I, I, C, P]),
            "or_linear": (None, [P, P, I, P, P, P, I, I, I, C, P, I, P, P]),
            "or_layout_bytes": (I, [I, I, C]),
            "or_relayout": (None, [P, P, P, I, I, C, P]),
            "or_interleave_word": (ctypes.c_uint32, [ctypes.c_uint32]),
            "or_f16_selfcheck": (I, [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- formats

def bf16_to_f32(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to fp32."""
    b = _c(bits, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def f32_to_f16_bits(x) -> np.ndarray:
    """IEEE binary16 round-to-nearest-even of fp32 values (the oracle's own
    conversion, written from the format definition)."""
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    _load().or_f32_to_f16_array(_ptr(x), _ptr(out), x.size)
    return out


def f16_bits_to_f64(h) -> np.ndarray:
    """Exact value of fp16 bit patterns (the oracle's own decoding)."""
    h = _c(h, np.uint16)
    out = np.empty(h.shape, np.float64)
    _load().or_f16_to_f64_array(_ptr(h), _ptr(out), h.size)
    return out


def round_half_even(v: float) -> float:
    return float(_load().or_round_half_even(float(v)))


def f16_selfcheck(start: int, stop: int, stride: int = 1) -> int:
    """Number of fp32 bit patterns start, start+stride, ... < stop where the
    oracle's fp16 conversion disagrees with the host compiler's _Float16 cast."""
    return int(_load().or_f16_selfcheck(start, stop, stride))


# ---------------------------------------------------------------- quantizer

def quantize_f32(w, group: int, bits: int = 4, sym: bool = False):
    """Per-group RTN of an fp32 matrix w [rows][cols] (groups of ``group``
    consecutive columns).  Returns (q int32 [rows][cols] signed codes,
    s16 uint16 [rows][cols/group], z16 uint16 or None, non-finite groups)."""
    w = _c(np.atleast_2d(w), np.float32)
    rows, cols = w.shape
    assert cols % group == 0
    q = np.empty((rows, cols), np.int32)
    s16 = np.empty((rows, cols // group), np.uint16)
    z16 = None if sym else np.empty((rows, cols // group), np.uint16)
    bad = _load().or_quantize_f32(_ptr(w), rows, cols, group, bits, int(sym),
                                  _ptr(q), _ptr(s16), _ptr(z16))
    return q, s16, z16, int(bad)


def awq_fold_weight(w, s) -> np.ndarray:
    """W' = W diag(s) in fp32 (one rounded product per element)."""
    w = _c(np.atleast_2d(w), np.float32)
    s = _c(s, np.float32)
    out = np.empty_like(w)
    _load().or_awq_fold_weight(_ptr(w), _ptr(s), w.shape[0], w.shape[1], _ptr(out))
    return out


def quantize_bf16(W_bits, awq_s=None, group: int = GROUP, sym: bool = False):
    """4-bit RTN of a bf16 weight matrix (uint16 bit patterns, [N][K]) with the
    optional AWQ per-input-channel scale folded in.  Same returns as
    :func:`quantize_f32`."""
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    s = None if awq_s is None else _c(awq_s, np.float32)
    q = np.empty((N, K), np.int32)
    s16 = np.empty((N, K // group), np.uint16)
    z16 = None if sym else np.empty((N, K // group), np.uint16)
    bad = _load().or_quantize_bf16(_ptr(W), _ptr(s), N, K, group, int(sym),
                                   _ptr(q), _ptr(s16), _ptr(z16))
    if bad < 0:
        raise MemoryError("oracle quantize: allocation failed")
    return q, s16, z16, int(bad)


def pack_u4(q, sym: bool) -> np.ndarray:
    q = _c(q, np.int32)
    N, K = q.shape
    P = np.empty((N, K // 8), np.uint32)
    _load().or_pack_u4(_ptr(q), N, K, int(sym), _ptr(P))
    return P


def unpack_u4(P, K: int, sym: bool) -> np.ndarray:
    P = _c(P, np.uint32)
    N = P.shape[0]
    q = np.empty((N, K), np.int32)
    _load().or_unpack_u4(_ptr(P), N, K, int(sym), _ptr(q))
    return q


def dequant(P, s16, z16, K: int, group: int = GROUP, sym: bool = False) -> np.ndarray:
    """x_hat = s16 (q - z16) in fp64 from the canonical packed words."""
    P = _c(P, np.uint32)
    N = P.shape[0]
    out = np.empty((N, K), np.float64)
    _load().or_dequant(_ptr(P), _ptr(_c(s16, np.uint16)),
                       None if sym else _ptr(_c(z16, np.uint16)), N, K, group, int(sym), _ptr(out))
    return out


def linear(x_bits, P, s16, z16, K: int, group: int = GROUP, sym: bool = False,
           awq_s=None, rows=None) -> np.ndarray:
    """y = x' dequant(W)^T in fp64.  x_bits: bf16 bit patterns [M][K];
    awq_s: the AWQ scale s (x' = x / s) or None; rows: output channels to
    compute (None = all).  Returns float64 [M][len(rows)]."""
    x = _c(np.atleast_2d(x_bits), np.uint16)
    M = x.shape[0]
    P = _c(P, np.uint32)
    N = P.shape[0]
    r = None if rows is None else _c(rows, np.int64)
    nrows = N if r is None else r.size
    y = np.empty((M, nrows), np.float64)
    scratch = np.empty(K, np.float64)
    s = None if awq_s is None else _c(awq_s, np.float32)
    _load().or_linear(_ptr(x), _ptr(s), M, _ptr(P), _ptr(_c(s16, np.uint16)),
                      None if sym else _ptr(_c(z16, np.uint16)), N, K, group, int(sym),
                      _ptr(r), nrows, _ptr(y), _ptr(scratch))
    return y


# ---------------------------------------------------------------- kernel layout

def layout_bytes(N: int, K: int, sym: bool) -> int:
    return int(_load().or_layout_bytes(N, K, int(sym)))


def interleave_word(w: int) -> int:
    """Nibble slot t of the result holds canonical nibble 2t (t < 4) or
    2(t-4)+1 (t >= 4)."""
    return int(_load().or_interleave_word(int(w)))


def relayout(P, s16, z16, N: int, K: int, sym: bool) -> np.ndarray:
    """The bytes of kernel layout 1 (tiled) for canonical (P, s16, z16)."""
    out = np.empty(layout_bytes(N, K, sym), np.uint8)
    _load().or_relayout(_ptr(_c(P, np.uint32)), _ptr(_c(s16, np.uint16)),
                        None if sym else _ptr(_c(z16, np.uint16)), N, K, int(sym), _ptr(out))
    return out
