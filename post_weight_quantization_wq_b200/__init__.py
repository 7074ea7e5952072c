"""B200-native 4-bit per-group (G=128) weight quantization and W4A16 decode linear.

The compute runs in ``libwq_b200.so`` (hand-written sm_100a CUDA behind the C
ABI of ``include/wq.h``); this package only allocates device buffers with
PyTorch and calls the ABI through :mod:`._binding`.  There is no CPU path:
every function here raises if the library or a GPU is missing.

    qw = quantize(W)                 # wq_quantize_rtn + wq_pack_layout
    y = linear(x, qw)                # wq_gemv_w4a16 (M <= 2, or with the AWQ factor) /
                                     # wq_gemm_w4a16 (tensor cores, M >= 3)
"""
from __future__ import annotations

from dataclasses import dataclass

from . import _binding as abi
from ._binding import WqError

GROUP = abi.WQ_GROUP_SIZE
LAYOUT = abi.WQ_LAYOUT_TILED


def _check(status: int, where: str) -> None:
    if status != abi.WQ_OK:
        raise WqError(status, where)


def _require(t, name: str, dtype, shape=None, device=None):
    """The C ABI takes raw device pointers: refuse anything it would misread
    (host memory, another dtype, a strided view, a wrong shape or GPU)."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor (got {t.device})")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


@dataclass
class QuantizedWeight:
    """A quantized weight: canonical buffers plus the kernel-layout copy."""
    N: int
    K: int
    symmetric: bool
    qweight: "object"        # torch.int32 [N][K/8] (uint32 words)
    scales: "object"         # torch.float16 [N][K/128]
    zeros: "object"          # torch.float16 [N][K/128] or None
    packed: "object"         # torch.uint8 [wq_packed_bytes]
    nonfinite_groups: int = 0


def quantize(W, awq_scale=None, symmetric: bool = False, stream=None,
             check_finite: bool = True) -> QuantizedWeight:
    """Quantize a bf16 CUDA tensor W [N][K] (optionally with the AWQ scale
    folded in) and lay it out for the linear kernels."""
    import torch
    if getattr(W, "dim", lambda: 0)() != 2:
        raise ValueError("W: expected a 2-D tensor [N][K]")
    N, K = W.shape
    _require(W, "W", torch.bfloat16)
    dev = W.device
    if awq_scale is not None:
        _require(awq_scale, "awq_scale", torch.float32, (K,), dev)
    qweight = torch.empty((N, K // 8), dtype=torch.int32, device=dev)
    scales = torch.empty((N, K // GROUP), dtype=torch.float16, device=dev)
    zeros = None if symmetric else torch.empty((N, K // GROUP), dtype=torch.float16, device=dev)
    d_status = torch.zeros(4, dtype=torch.int32, device=dev)
    _check(abi.wq_quantize_rtn(W, awq_scale, N, K, GROUP, symmetric, qweight, scales, zeros,
                               d_status, stream), "wq_quantize_rtn")
    nbytes = abi.wq_packed_bytes(N, K, GROUP, symmetric, LAYOUT)
    packed = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(abi.wq_pack_layout(qweight, scales, zeros, N, K, GROUP, symmetric, LAYOUT, packed,
                              nbytes, stream), "wq_pack_layout")
    bad = int(d_status[0].item()) if check_finite else 0
    return QuantizedWeight(N, K, symmetric, qweight, scales, zeros, packed, bad)


def gptq_quantize(W, X, symmetric: bool = False, damp: float = 0.01, stream=None,
                  workspace=None) -> QuantizedWeight:
    """GPTQ on the GPU (wq_gptq_quantize): bf16 CUDA tensors W [N][K] and
    calibration inputs X [T][K]; returns the same QuantizedWeight as
    quantize(), laid out for the linears.  nonfinite_groups holds the
    device status word (0 when all went well)."""
    import torch
    if getattr(W, "dim", lambda: 0)() != 2 or getattr(X, "dim", lambda: 0)() != 2:
        raise ValueError("W [N][K] and X [T][K] must be 2-D")
    N, K = W.shape
    T = X.shape[0]
    _require(W, "W", torch.bfloat16)
    _require(X, "X", torch.bfloat16, (T, K), W.device)
    dev = W.device
    qweight = torch.empty((N, K // 8), dtype=torch.int32, device=dev)
    scales = torch.empty((N, K // GROUP), dtype=torch.float16, device=dev)
    zeros = None if symmetric else torch.empty((N, K // GROUP), dtype=torch.float16, device=dev)
    need = abi.wq_gptq_workspace_bytes(T, N, K)
    if need == 0:
        raise ValueError(f"gptq_quantize: unsupported sizes T={T} N={N} K={K}")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    d_status = torch.zeros(4, dtype=torch.int32, device=dev)
    _check(abi.wq_gptq_quantize(W, X, T, N, K, GROUP, symmetric, damp, qweight, scales, zeros,
                                workspace, workspace.numel(), d_status, stream),
           "wq_gptq_quantize")
    nbytes = abi.wq_packed_bytes(N, K, GROUP, symmetric, LAYOUT)
    packed = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(abi.wq_pack_layout(qweight, scales, zeros, N, K, GROUP, symmetric, LAYOUT, packed,
                              nbytes, stream), "wq_pack_layout")
    return QuantizedWeight(N, K, symmetric, qweight, scales, zeros, packed,
                           int(d_status[0].item()))


def awq_search(W, X, symmetric: bool = False, n_grid: int = 20, stream=None, workspace=None):
    """AWQ scale search on the GPU (wq_awq_search): bf16 CUDA tensors W [N][K]
    and calibration inputs X [T][K].  Returns a dict with the fp64 losses of
    every alpha = i / n_grid (host numpy), the chosen index ``i`` and
    ``alpha``, and ``s`` (fp32 CUDA tensor [K]) to pass to quantize() as
    awq_scale (and 1/s to linear() as inv_act_scale)."""
    import torch
    if getattr(W, "dim", lambda: 0)() != 2 or getattr(X, "dim", lambda: 0)() != 2:
        raise ValueError("W [N][K] and X [T][K] must be 2-D")
    N, K = W.shape
    T = X.shape[0]
    _require(W, "W", torch.bfloat16)
    _require(X, "X", torch.bfloat16, (T, K), W.device)
    dev = W.device
    need = abi.wq_awq_search_workspace_bytes(T, N, K, n_grid)
    if need == 0:
        raise ValueError(f"awq_search: unsupported sizes T={T} N={N} K={K} n_grid={n_grid}")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    losses = torch.empty(n_grid + 1, dtype=torch.float64, device=dev)
    s = torch.empty(K, dtype=torch.float32, device=dev)
    best = torch.zeros(4, dtype=torch.int32, device=dev)
    _check(abi.wq_awq_search(W, X, T, N, K, GROUP, symmetric, n_grid, losses, s, best, workspace,
                             workspace.numel(), stream), "wq_awq_search")
    i = int(best[0].item())
    return {"losses": losses.cpu().numpy(), "i": i, "alpha": i / n_grid, "s": s}


@dataclass
class Nvfp4Weight:
    """An NVFP4 weight: canonical codes / block scales / tensor scale plus the
    layout the FP4 tensor-core linear reads."""
    N: int
    K: int
    codes: "object"          # torch.uint8 [N][K/2]
    scales: "object"         # torch.uint8 [N][K/16] (E4M3)
    tensor_scale: "object"   # torch.float32 [1]
    packed: "object"         # torch.uint8 [wq_nvfp4_packed_bytes]
    nonfinite: int = 0


def nvfp4_quantize_tensor(A, stream=None):
    """NVFP4 codes, E4M3 block scales and the fp32 tensor scale of a bf16 CUDA
    tensor A [R][C] (wq_nvfp4_quantize)."""
    import torch
    R, C = A.shape
    _require(A, "A", torch.bfloat16)
    codes = torch.empty((R, C // 2), dtype=torch.uint8, device=A.device)
    scales = torch.empty((R, C // 16), dtype=torch.uint8, device=A.device)
    S = torch.empty(4, dtype=torch.float32, device=A.device)
    d_status = torch.zeros(4, dtype=torch.int32, device=A.device)
    _check(abi.wq_nvfp4_quantize(A, R, C, codes, scales, S, d_status, stream), "wq_nvfp4_quantize")
    return codes, scales, S, d_status


def nvfp4_quantize(W, stream=None) -> Nvfp4Weight:
    """Quantize a bf16 CUDA weight W [N][K] to NVFP4 and lay it out for
    nvfp4_linear()."""
    import torch
    N, K = W.shape
    codes, scales, S, d_status = nvfp4_quantize_tensor(W, stream)
    nbytes = abi.wq_nvfp4_packed_bytes(N, K)
    packed = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    _check(abi.wq_nvfp4_pack_layout(codes, scales, N, K, packed, nbytes, stream),
           "wq_nvfp4_pack_layout")
    return Nvfp4Weight(N, K, codes, scales, S, packed, int(d_status[0].item()))


def nvfp4_linear(x, qw: Nvfp4Weight, out=None, workspace=None, stream=None):
    """y = dequant(nvfp4(x)) dequant(W)^T as fp32 [M][N] on the FP4 tensor
    cores (wq_nvfp4_linear); x bf16 CUDA [M][K], M <= 128."""
    import torch
    M, K = x.shape
    _require(x, "x", torch.bfloat16, (M, qw.K), qw.packed.device)
    y = out if out is not None else torch.empty((M, qw.N), dtype=torch.float32, device=x.device)
    need = abi.wq_nvfp4_linear_workspace_bytes(M, qw.N, K)
    if need == 0:
        raise ValueError(f"nvfp4_linear: unsupported sizes M={M} N={qw.N} K={K}")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _check(abi.wq_nvfp4_linear(x, qw.packed, qw.tensor_scale, M, qw.N, K, y, workspace,
                               workspace.numel(), stream), "wq_nvfp4_linear")
    return y


_workspaces = {}


def workspace_for(M: int, N: int, K: int, device, path: str = "gemv", stream=None):
    """A zero-filled workspace large enough for (M, N, K) on the given path,
    cached per (device, stream) -- calls that share a workspace must not run
    concurrently -- and only ever grown."""
    import torch
    need = abi.wq_gemm_workspace_bytes(M, N, K) if path == "gemm" else \
        abi.wq_workspace_bytes(M, N, K)
    if need == 0:
        return None, 0
    key = (str(device), abi._stream(stream))
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(need, dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws, ws.numel()


GEMV_MAX_ROWS = 2


def linear(x, qw: QuantizedWeight, inv_act_scale=None, out=None, workspace=None, stream=None,
           path=None):
    """y = x' dequant(W)^T as fp32 [M][N] for a bf16 CUDA tensor x [M][K].
    path: None (choose by M), "gemv" (wq_gemv_w4a16, M <= 8) or "gemm"
    (wq_gemm_w4a16, tensor cores, no AWQ factor)."""
    import torch
    if getattr(x, "dim", lambda: 0)() != 2:
        raise ValueError("x: expected a 2-D tensor [M][K]")
    M, K = x.shape
    _require(x, "x", torch.bfloat16, (M, qw.K), qw.packed.device)
    if inv_act_scale is not None:
        _require(inv_act_scale, "inv_act_scale", torch.float32, (K,), x.device)
    if out is not None:
        _require(out, "out", torch.float32, (M, qw.N), x.device)
    if workspace is not None:
        _require(workspace, "workspace", torch.uint8, None, x.device)
    y = out if out is not None else torch.empty((M, qw.N), dtype=torch.float32, device=x.device)
    # wq_gemv_w4a16 up to 2 rows and for the AWQ fold (its scaled activations
    # are not exact in a bf16 tensor-core operand); wq_gemm_w4a16 from 3 rows
    # on.  Both entries run the int8 tensor-core kernel where it applies
    # (K a multiple of 512: M = 2..8 / M <= 16); otherwise the bf16 skinny
    # GEMM beats the CUDA-core GEMV from about M = 3.
    if path is None:
        path = "gemv" if (M <= GEMV_MAX_ROWS or inv_act_scale is not None) else "gemm"
    if workspace is None:
        ws, ws_bytes = workspace_for(M, qw.N, K, x.device, path, stream)
    else:
        ws, ws_bytes = workspace, workspace.numel()
    fn = abi.wq_gemv_w4a16 if path == "gemv" else abi.wq_gemm_w4a16
    _check(fn(x, inv_act_scale, qw.packed, M, qw.N, K, GROUP, qw.symmetric, LAYOUT, y, ws,
              ws_bytes, stream), fn.__name__)
    return y


def reset_workspaces(device=None) -> None:
    """Forget the cached workspaces (of one device, or all); the next call
    allocates a fresh zero-filled one."""
    for key in list(_workspaces):
        if device is None or key[0] == str(device):
            del _workspaces[key]


def last_device_status(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device error word
    (wq_last_device_status).  A call cut short by a bounded-wait timeout may
    leave split-K completion counters set in its workspace, so on
    WQ_ERR_TIMEOUT the cached workspaces of the current device are dropped:
    later linear() calls without an explicit workspace start from zeroed
    ones.  A caller-owned workspace must be zeroed by the caller."""
    import torch
    st = abi.wq_last_device_status(stream)
    if st == abi.WQ_ERR_TIMEOUT:
        reset_workspaces(torch.device("cuda", torch.cuda.current_device()))
    return st
