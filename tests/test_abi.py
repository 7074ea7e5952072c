"""The C-ABI library loads and exports every function include/wq.h declares,
and its host-side logic (sizes, validation that returns before any launch)
behaves as documented.  No CUDA work is enqueued here."""
import os
import re

import pytest

from post_weight_quantization_wq_b200 import _binding as abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(wq_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = abi.load()
    declared = _declared_functions()
    assert "wq_gemv_w4a16" in declared and "wq_quantize_rtn" in declared
    for name in declared:
        assert hasattr(lib, name), name
        assert name in abi.SIGNATURES, name


def test_abi_version_and_status_strings():
    assert abi.wq_abi_version() == 1
    assert abi.status_string(abi.WQ_OK) == "WQ_OK"
    assert abi.status_string(abi.WQ_ERR_TIMEOUT) == "WQ_ERR_TIMEOUT"
    assert abi.status_string(99) == "WQ_ERR_UNKNOWN"


def test_packed_bytes_matches_layout_definition():
    import oracle
    for N, K, sym in [(256, 1024, 0), (4096, 11008, 1), (200, 640, 0), (1, 128, 1),
                      (28672, 8192, 0), (8192, 28672, 0)]:
        assert abi.wq_packed_bytes(N, K, 128, sym, 1) == oracle.layout_bytes(N, K, bool(sym))
    assert abi.wq_packed_bytes(256, 1000, 128, 0, 1) == 0
    assert abi.wq_packed_bytes(256, 1024, 64, 0, 1) == 0
    assert abi.wq_packed_bytes(256, 1024, 128, 0, 2) == 0
    assert abi.wq_packed_bytes(0, 1024, 128, 0, 1) == 0


def test_workspace_bytes():
    C = abi.WQ_WORKSPACE_COUNTER_BYTES
    # GEMV, CUDA-core shapes (M = 1, or K not a multiple of 512): one slab
    # needs no workspace; otherwise counters + partials [slabs][padded M][Npad]
    assert abi.wq_workspace_bytes(1, 4096, 512) == 0
    assert abi.wq_workspace_bytes(2, 4096, 384) == 0
    assert abi.wq_workspace_bytes(2, 4096, 640) == C + 2 * 2 * 4096 * 4
    assert abi.wq_workspace_bytes(1, 8192, 28672) == C + 56 * 1 * 8192 * 4
    assert abi.wq_workspace_bytes(5, 8192, 28288) == C + 56 * 8 * 8192 * 4
    # GEMV, tensor-core shapes (M = 2..8, K a multiple of 512): the same
    # prefix, then the prepared activation rows per slab (4 K-blocks x 2 Mpad
    # rows x 128 B) and the chunk factors (Mpad x 8 float2), each padded to 256 B
    assert abi.wq_workspace_bytes(2, 4096, 512) == C + 2048 + 256
    assert abi.wq_workspace_bytes(3, 8192, 28672) == (C + 56 * 4 * 8192 * 4 + 56 * 4096
                                                      + 56 * 256)
    assert abi.wq_workspace_bytes(5, 8192, 28672) == (C + 56 * 8 * 8192 * 4 + 56 * 8192
                                                      + 56 * 512)
    # GEMM: counters, partials padded to 16-row multiples, sum(x) per group
    # (M <= 16 with K a multiple of 512: the largest of that and the int8
    # kernel's, whose prepared rows take 4 x 2 Mpad x 128 B and chunk
    # factors Mpad x 64 B per slab)
    gemm16 = C + 56 * 16 * 8192 * 4 + 224 * 64 * 4
    tc16 = C + 56 * 16 * 8192 * 4 + 56 * 16384 + 56 * 1024
    assert abi.wq_gemm_workspace_bytes(1, 4096, 512) == C + 2048 + 256
    assert abi.wq_gemm_workspace_bytes(1, 4096, 1408) == C + 3 * 16 * 4096 * 4 + 11 * 64 * 4
    assert abi.wq_gemm_workspace_bytes(1, 8192, 28672) == gemm16
    assert abi.wq_gemm_workspace_bytes(16, 8192, 28672) == tc16
    assert abi.wq_gemm_workspace_bytes(17, 8192, 28672) == C + 56 * 32 * 8192 * 4 + 224 * 64 * 4
    assert abi.wq_workspace_bytes(9, 8192, 28672) == tc16           # M = 9..64: GEMM only
    assert abi.wq_workspace_bytes(64, 8192, 28672) == abi.wq_gemm_workspace_bytes(64, 8192, 28672)
    assert abi.wq_workspace_bytes(0, 8192, 8192) == 0
    # M > 64: the many-row kernel's sums of x [groups][rows padded to 128]
    # (plus split-K partials when the shape needs them)
    assert abi.wq_gemm_workspace_bytes(512, 28672, 8192) == C + 64 * 512 * 4
    assert abi.wq_gemm_workspace_bytes(65, 8192, 8192) >= C + 64 * 128 * 4
    assert abi.wq_workspace_bytes(65, 8192, 8192) == abi.wq_gemm_workspace_bytes(65, 8192, 8192)
    assert abi.wq_gemm_workspace_bytes(abi.WQ_GEMM_MAX_M + 1, 8192, 8192) == 0
    assert abi.wq_workspace_bytes(1, 8192, 100) == 0          # K not a multiple of 128


@pytest.mark.parametrize("args,expect", [
    (dict(N=0), abi.WQ_ERR_INVALID_ARG),
    (dict(K=1000), abi.WQ_ERR_UNSUPPORTED_SHAPE),
    (dict(group_size=64), abi.WQ_ERR_UNSUPPORTED_SHAPE),
    (dict(N=1 << 21), abi.WQ_ERR_UNSUPPORTED_SHAPE),
    (dict(symmetric=2), abi.WQ_ERR_INVALID_ARG),
    (dict(W=0), abi.WQ_ERR_INVALID_ARG),
    (dict(zeros=0), abi.WQ_ERR_INVALID_ARG),              # asymmetric needs zeros
    (dict(symmetric=1), abi.WQ_ERR_INVALID_ARG),          # symmetric forbids zeros
    (dict(W=0x1008), abi.WQ_ERR_MISALIGNED),
])
def test_quantize_validation_before_launch(args, expect):
    a = dict(W=0x1000, awq=None, N=256, K=1024, group_size=128, symmetric=0, qweight=0x2000,
             scales=0x3000, zeros=0x4000, d_status=None)
    a.update(args)
    st = abi.wq_quantize_rtn(a["W"] or None, a["awq"], a["N"], a["K"], a["group_size"],
                             a["symmetric"], a["qweight"], a["scales"], a["zeros"] or None,
                             a["d_status"], 0)
    assert st == expect


@pytest.mark.parametrize("fn,M", [("wq_gemv_w4a16", 0), ("wq_gemv_w4a16", 9),
                                  ("wq_gemm_w4a16", 0),
                                  ("wq_gemm_w4a16", abi.WQ_GEMM_MAX_M + 1)])
def test_linear_rejects_m_out_of_range(fn, M):
    st = getattr(abi, fn)(0x1000, None, 0x2000, M, 256, 1024, 128, 0, 1, 0x3000, 0x4000,
                          1 << 30, 0)
    assert st == abi.WQ_ERR_UNSUPPORTED_SHAPE


def test_linear_validation_before_launch():
    call = abi.wq_gemv_w4a16
    base = (0x1000, None, 0x2000, 1, 8192, 28672, 128, 0, 1, 0x3000, 0x4000, 1 << 30, 0)
    # misaligned x
    a = list(base); a[0] = 0x1004
    assert call(*a) == abi.WQ_ERR_MISALIGNED
    # workspace too small / missing
    a = list(base); a[11] = 100
    assert call(*a) == abi.WQ_ERR_WORKSPACE_TOO_SMALL
    a = list(base); a[10] = None
    assert call(*a) == abi.WQ_ERR_WORKSPACE_TOO_SMALL
    # unknown layout, NULL y
    a = list(base); a[8] = 7
    assert call(*a) == abi.WQ_ERR_INVALID_ARG
    a = list(base); a[9] = None
    assert call(*a) == abi.WQ_ERR_INVALID_ARG
    # the tensor-core path takes no activation scale
    a = list(base); a[1] = 0x5000; a[3] = 16
    assert abi.wq_gemm_w4a16(*a) == abi.WQ_ERR_INVALID_ARG


def test_pack_layout_validation_before_launch():
    st = abi.wq_pack_layout(0x1000, 0x2000, 0x3000, 256, 1024, 128, 0, 1, 0x4000, 10, 0)
    assert st == abi.WQ_ERR_INVALID_ARG        # packed buffer too small
    st = abi.wq_pack_layout(0x1000, 0x2000, None, 256, 1024, 128, 0, 1, 0x4000, 1 << 20, 0)
    assert st == abi.WQ_ERR_INVALID_ARG        # asymmetric needs zeros


def test_static_gemv_validation_before_launch():
    """The allocation-free GEMV refuses, before touching the GPU, shapes whose
    scratch exceeds its static array, and bad arguments."""
    assert abi.wq_workspace_bytes(8, 8192, 28672) > abi.WQ_STATIC_SCRATCH_BYTES
    st = abi.wq_gemv_w4a16_static(0x1000, None, 0x2000, 8, 8192, 28672, 128, 0, 1, 0x3000, 0)
    assert st == abi.WQ_ERR_WORKSPACE_TOO_SMALL
    st = abi.wq_gemv_w4a16_static(0x1000, None, 0x2000, 9, 8192, 28672, 128, 0, 1, 0x3000, 0)
    assert st == abi.WQ_ERR_UNSUPPORTED_SHAPE
    st = abi.wq_gemv_w4a16_static(0x1004, None, 0x2000, 1, 256, 1024, 128, 0, 1, 0x3000, 0)
    assert st == abi.WQ_ERR_MISALIGNED


def test_stream_read_probe_validation_before_launch():
    # argument errors are reported before any CUDA call (no GPU needed)
    assert abi.wq_stream_read_probe(None, 1024, 64, 0) == abi.WQ_ERR_INVALID_ARG
    assert abi.wq_stream_read_probe(256, 0, 64, 0) == abi.WQ_ERR_INVALID_ARG
    assert abi.wq_stream_read_probe(256, 1000, 64, 0) == abi.WQ_ERR_INVALID_ARG
    assert abi.wq_stream_read_probe(256, 1024, None, 0) == abi.WQ_ERR_INVALID_ARG
    assert abi.wq_stream_read_probe(264, 1024, 64, 0) == abi.WQ_ERR_MISALIGNED
    assert abi.wq_stream_read_probe(256, 1024, 66, 0) == abi.WQ_ERR_MISALIGNED
