"""The read-bandwidth probe reads every byte: its XOR checksum equals the
XOR of the buffer's 32-bit words computed on the host."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nbytes", [16, 4096, (1 << 20) + 48, 64 << 20])
def test_stream_read_probe_checksum(nbytes):
    import torch
    from post_weight_quantization_wq_b200 import _binding as abi
    words = np.random.default_rng(nbytes).integers(0, 2**32, size=nbytes // 4, dtype=np.uint32)
    buf = torch.from_numpy(words.view(np.int32)).cuda()
    out = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    assert abi.wq_stream_read_probe(buf, nbytes, out) == 0
    torch.cuda.synchronize()
    assert np.uint32(out.item() & 0xFFFFFFFF) == np.bitwise_xor.reduce(words)
    assert abi.wq_last_device_status() == 0
