"""ctypes binding of ``libwq_b200.so`` (the C ABI in ``include/wq.h``).

Argument marshalling only: each function has the name and the arguments of
its C counterpart; tensors are passed as their device pointers, streams as
``torch.cuda.Stream`` (or a raw handle, or None for the current stream).
Every step of the computation runs in the library's CUDA kernels.  Loading
fails loudly when the library is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libwq_b200.so")

WQ_OK = 0
WQ_ERR_INVALID_ARG = 1
WQ_ERR_UNSUPPORTED_SHAPE = 2
WQ_ERR_MISALIGNED = 3
WQ_ERR_WORKSPACE_TOO_SMALL = 4
WQ_ERR_NONFINITE = 5
WQ_ERR_TIMEOUT = 6
WQ_ERR_CUDA = 7
WQ_GROUP_SIZE = 128
WQ_LAYOUT_TILED = 1
WQ_WORKSPACE_COUNTER_BYTES = 262144
WQ_STATIC_SCRATCH_BYTES = 8 << 20
WQ_GPTQ_MAX_K = 32768
WQ_GPTQ_MAX_T = 65536
WQ_AWQ_MAX_T = 65536
WQ_AWQ_MAX_GRID = 1000
WQ_NVFP4_MAX_M = 128
WQ_GEMM_MAX_M = 65536

# name -> (restype, argtypes); the exported symbols of include/wq.h
_P = ctypes.c_void_p
_I = ctypes.c_int
_S = ctypes.c_size_t
SIGNATURES = {
    "wq_status_string": (ctypes.c_char_p, [_I]),
    "wq_abi_version": (_I, []),
    "wq_quantize_rtn": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P]),
    "wq_packed_bytes": (_S, [_I, _I, _I, _I, _I]),
    "wq_pack_layout": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _S, _P]),
    "wq_workspace_bytes": (_S, [_I, _I, _I]),
    "wq_gemm_workspace_bytes": (_S, [_I, _I, _I]),
    "wq_gemv_w4a16": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _S, _P]),
    "wq_gemm_w4a16": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _S, _P]),
    "wq_gemv_w4a16_static": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P]),
    "wq_last_device_status": (_I, [_P]),
    "wq_debug_set_wait_limit_ns": (None, [ctypes.c_ulonglong]),
    "wq_debug_gemm_force_fold": (None, [_I]),
    "wq_debug_gemv_force_cuda_cores": (None, [_I]),
    "wq_stream_read_probe": (_I, [_P, _S, _P, _P]),
    "wq_debug_gemv_split": (_I, [_I, _I, _I, _I, _I, _I, _P, _P, _P]),
    "wq_gptq_workspace_bytes": (_S, [_I, _I, _I]),
    "wq_awq_search_workspace_bytes": (_S, [_I, _I, _I, _I]),
    "wq_nvfp4_quantize": (_I, [_P, _I, _I, _P, _P, _P, _P, _P]),
    "wq_nvfp4_packed_bytes": (_S, [_I, _I]),
    "wq_nvfp4_pack_layout": (_I, [_P, _P, _I, _I, _P, _S, _P]),
    "wq_nvfp4_linear_workspace_bytes": (_S, [_I, _I, _I]),
    "wq_nvfp4_linear": (_I, [_P, _P, _P, _I, _I, _I, _P, _P, _S, _P]),
    "wq_awq_search": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _S, _P]),
    "wq_gptq_quantize": (_I, [_P, _P, _I, _I, _I, _I, _I, ctypes.c_double, _P, _P, _P, _P, _S,
                              _P, _P]),
}

_lock = threading.Lock()
_lib = None


class WqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (once).  Raises if it is missing."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise ImportError(
                f"libwq_b200.so not found at {path}; build it with "
                "`python -m post_weight_quantization_wq_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def status_string(status: int) -> str:
    return load().wq_status_string(int(status)).decode()


def wq_abi_version() -> int:
    return load().wq_abi_version()


def wq_quantize_rtn(W, awq_scale, N, K, group_size, symmetric, qweight, scales, zeros,
                    d_status, stream=None) -> int:
    return load().wq_quantize_rtn(_ptr(W), _ptr(awq_scale), N, K, group_size, int(symmetric),
                                  _ptr(qweight), _ptr(scales), _ptr(zeros), _ptr(d_status),
                                  _stream(stream))


def wq_packed_bytes(N, K, group_size, symmetric, layout) -> int:
    return load().wq_packed_bytes(N, K, group_size, int(symmetric), layout)


def wq_pack_layout(qweight, scales, zeros, N, K, group_size, symmetric, layout, packed,
                   packed_bytes, stream=None) -> int:
    return load().wq_pack_layout(_ptr(qweight), _ptr(scales), _ptr(zeros), N, K, group_size,
                                 int(symmetric), layout, _ptr(packed), packed_bytes,
                                 _stream(stream))


def wq_workspace_bytes(M, N, K) -> int:
    return load().wq_workspace_bytes(M, N, K)


def wq_gemm_workspace_bytes(M, N, K) -> int:
    return load().wq_gemm_workspace_bytes(M, N, K)


def wq_gemv_w4a16(x, inv_act_scale, packed, M, N, K, group_size, symmetric, layout, y,
                  workspace, ws_bytes, stream=None) -> int:
    return load().wq_gemv_w4a16(_ptr(x), _ptr(inv_act_scale), _ptr(packed), M, N, K,
                                group_size, int(symmetric), layout, _ptr(y), _ptr(workspace),
                                ws_bytes, _stream(stream))


def wq_gemm_w4a16(x, inv_act_scale, packed, M, N, K, group_size, symmetric, layout, y,
                  workspace, ws_bytes, stream=None) -> int:
    return load().wq_gemm_w4a16(_ptr(x), _ptr(inv_act_scale), _ptr(packed), M, N, K,
                                group_size, int(symmetric), layout, _ptr(y), _ptr(workspace),
                                ws_bytes, _stream(stream))


def wq_gemv_w4a16_static(x, inv_act_scale, packed, M, N, K, group_size, symmetric, layout, y,
                         stream=None) -> int:
    return load().wq_gemv_w4a16_static(_ptr(x), _ptr(inv_act_scale), _ptr(packed), M, N, K,
                                       group_size, int(symmetric), layout, _ptr(y),
                                       _stream(stream))


def wq_last_device_status(stream=None) -> int:
    return load().wq_last_device_status(_stream(stream))


def wq_debug_set_wait_limit_ns(ns: int) -> None:
    load().wq_debug_set_wait_limit_ns(int(ns))


def wq_debug_gemm_force_fold(on: int) -> None:
    load().wq_debug_gemm_force_fold(int(on))


def wq_debug_gemv_force_cuda_cores(on: int) -> None:
    load().wq_debug_gemv_force_cuda_cores(int(on))


def wq_debug_gemv_split(M, N, K, awq, num_sms, ctas_per_sm):
    """(status, tiles, teams per CTA, grid CTAs) of wq_gemv_w4a16's split."""
    tiles, teams, grid = ctypes.c_longlong(), ctypes.c_int(), ctypes.c_longlong()
    st = load().wq_debug_gemv_split(M, N, K, int(awq), num_sms, ctas_per_sm, ctypes.byref(tiles),
                                    ctypes.byref(teams), ctypes.byref(grid))
    return st, tiles.value, teams.value, grid.value


def wq_stream_read_probe(buf, nbytes, out, stream=None) -> int:
    return load().wq_stream_read_probe(_ptr(buf), int(nbytes), _ptr(out), _stream(stream))


def wq_gptq_workspace_bytes(T, N, K) -> int:
    return load().wq_gptq_workspace_bytes(T, N, K)


def wq_gptq_quantize(W, X, T, N, K, group_size, symmetric, damp, qweight, scales, zeros,
                     workspace, ws_bytes, d_status, stream=None) -> int:
    return load().wq_gptq_quantize(_ptr(W), _ptr(X), T, N, K, group_size, int(symmetric),
                                   float(damp), _ptr(qweight), _ptr(scales), _ptr(zeros),
                                   _ptr(workspace), ws_bytes, _ptr(d_status), _stream(stream))


def wq_awq_search_workspace_bytes(T, N, K, n_grid) -> int:
    return load().wq_awq_search_workspace_bytes(T, N, K, n_grid)


def wq_awq_search(W, X, T, N, K, group_size, symmetric, n_grid, losses, scale_out, best,
                  workspace, ws_bytes, stream=None) -> int:
    return load().wq_awq_search(_ptr(W), _ptr(X), T, N, K, group_size, int(symmetric), n_grid,
                                _ptr(losses), _ptr(scale_out), _ptr(best), _ptr(workspace),
                                ws_bytes, _stream(stream))


def wq_nvfp4_quantize(A, R, C, codes, block_scales, tensor_scale, d_status, stream=None) -> int:
    return load().wq_nvfp4_quantize(_ptr(A), R, C, _ptr(codes), _ptr(block_scales),
                                    _ptr(tensor_scale), _ptr(d_status), _stream(stream))


def wq_nvfp4_packed_bytes(N, K) -> int:
    return load().wq_nvfp4_packed_bytes(N, K)


def wq_nvfp4_pack_layout(codes, block_scales, N, K, packed, packed_bytes, stream=None) -> int:
    return load().wq_nvfp4_pack_layout(_ptr(codes), _ptr(block_scales), N, K, _ptr(packed),
                                       packed_bytes, _stream(stream))


def wq_nvfp4_linear_workspace_bytes(M, N, K) -> int:
    return load().wq_nvfp4_linear_workspace_bytes(M, N, K)


def wq_nvfp4_linear(x, packed, w_tensor_scale, M, N, K, y, workspace, ws_bytes,
                    stream=None) -> int:
    return load().wq_nvfp4_linear(_ptr(x), _ptr(packed), _ptr(w_tensor_scale), M, N, K, _ptr(y),
                                  _ptr(workspace), ws_bytes, _stream(stream))
