"""The allocation-free GEMV entry point (wq_gemv_w4a16_static) against the
workspace one (wq_gemv_w4a16), called through the C ABI.

wq_gemv_w4a16_static exists for callers that cannot allocate device memory
(a custom-op hook or plugin whose host forbids or owns every device
allocation, or a captured region with a fixed memory pool): it keeps its
split-K scratch in a static array inside the library.  Two calls in a row
must each reproduce the workspace entry point's output within the tolerance
the parity tests use (and in fact bit for bit: it is the same kernel with
the same fixed reduction order), and a repeated call must take no device
memory.  This file is collected last on purpose."""
import numpy as np
import pytest

from post_weight_quantization_wq_b200 import _binding as abi
from post_weight_quantization_wq_b200 import inputs

REL_L2 = 1e-3
MAX_ABS = 1e-2

pytestmark = pytest.mark.gpu


def _close(y, yref):
    y = y.astype(np.float64)
    yref = yref.astype(np.float64)
    err = y - yref
    assert np.linalg.norm(err) <= REL_L2 * np.linalg.norm(yref)
    assert np.max(np.abs(err)) <= MAX_ABS * np.sqrt(np.mean(yref ** 2))


@pytest.mark.parametrize("N,K,M,awq", [(8192, 28672, 1, False), (1024, 8192, 4, False),
                                       (300, 1408, 3, False), (2048, 4096, 1, True)])
def test_static_scratch_gemv_matches_workspace_gemv(N, K, M, awq):
    import torch
    import post_weight_quantization_wq_b200 as wq
    W = inputs.weights(N, K, 0.015, seed=N + K + M)
    Wt = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16)
    inv = None
    s = None
    if awq:
        s = np.exp(np.random.default_rng(M).uniform(-1, 1, K)).astype(np.float32)
        inv = torch.from_numpy((1.0 / s).astype(np.float32)).cuda()
    qw = wq.quantize(Wt, None if s is None else torch.from_numpy(s).cuda(), symmetric=False)
    x = torch.from_numpy(inputs.activations(M, K, seed=K + M).view(np.int16)).cuda().view(
        torch.bfloat16)

    ws_bytes = abi.wq_workspace_bytes(M, N, K)
    assert ws_bytes <= abi.WQ_STATIC_SCRATCH_BYTES
    ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    y_ref = torch.empty((M, N), dtype=torch.float32, device="cuda")
    assert abi.wq_gemv_w4a16(x, inv, qw.packed, M, N, K, 128, 0, 1, y_ref, ws, ws_bytes) == 0
    torch.cuda.synchronize()
    y_ref = y_ref.cpu().numpy()

    ys = [torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda") for _ in range(2)]
    for i, y in enumerate(ys):
        torch.cuda.synchronize()
        free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        assert abi.wq_gemv_w4a16_static(x, inv, qw.packed, M, N, K, 128, 0, 1, y) == 0
        assert abi.wq_last_device_status() == 0
        if i > 0:
            # after the first call (which may load the kernel), a call takes
            # no device memory at all
            assert torch.cuda.mem_get_info()[0] == free0
            assert torch.cuda.memory_allocated() == alloc0
        out = y.cpu().numpy()
        _close(out, y_ref)
        # the same kernel with the same fixed reduction order: bit-identical
        assert np.array_equal(out, y_ref)


def test_static_scratch_after_a_timeout():
    """A call cut short by a bounded-wait timeout may leave completion
    counters set in the static array; the next call clears the ones it uses
    itself, so it needs no help from the caller."""
    import torch
    import post_weight_quantization_wq_b200 as wq
    N, K, M = 4096, 8192, 1
    W = inputs.weights(N, K, 0.015, seed=77)
    qw = wq.quantize(torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16))
    x = torch.from_numpy(inputs.activations(M, K, seed=78).view(np.int16)).cuda().view(
        torch.bfloat16)
    ws_bytes = abi.wq_workspace_bytes(M, N, K)
    ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    y_ref = torch.empty((M, N), dtype=torch.float32, device="cuda")
    assert abi.wq_gemv_w4a16(x, None, qw.packed, M, N, K, 128, 0, 1, y_ref, ws, ws_bytes) == 0
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    try:
        abi.wq_debug_set_wait_limit_ns(1)
        for _ in range(3):
            assert abi.wq_gemv_w4a16_static(x, None, qw.packed, M, N, K, 128, 0, 1, y) == 0
        st = abi.wq_last_device_status()
    finally:
        abi.wq_debug_set_wait_limit_ns(2_000_000_000)
    assert st == abi.WQ_ERR_TIMEOUT
    for _ in range(2):
        y.fill_(float("nan"))
        assert abi.wq_gemv_w4a16_static(x, None, qw.packed, M, N, K, 128, 0, 1, y) == 0
        assert abi.wq_last_device_status() == 0
        assert torch.equal(y, y_ref)


def test_static_scratch_refuses_shapes_beyond_its_size():
    import torch
    # M = 8 on 8192 x 28672 needs 14.9 MB of partial sums: more than the array
    assert abi.wq_workspace_bytes(8, 8192, 28672) > abi.WQ_STATIC_SCRATCH_BYTES
    buf = torch.zeros(64, dtype=torch.uint8, device="cuda")
    st = abi.wq_gemv_w4a16_static(buf, None, buf, 8, 8192, 28672, 128, 0, 1, buf)
    assert st == abi.WQ_ERR_WORKSPACE_TOO_SMALL
