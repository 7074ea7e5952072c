"""Pins of the oracle's kernel-layout permutation (layout 1, "tiled").

The layout is this library's own format, not the pages': tiles of 128 rows x
one K-slab of 4 groups, slab-major; inside a tile the codes (row r at
r*gs*64 bytes, each word's nibbles interleaved so that slots t and t+4 hold
inputs 2t and 2t+1) then the metadata (entry (r, g) at (r*gs + g) * meta
bytes).  The offsets below are worked out by hand from that statement.
"""
import numpy as np
import pytest

import oracle


def _canonical(N, K):
    NG = K // 128
    P = ((np.arange(N, dtype=np.uint32)[:, None] << 16) |
         np.arange(K // 8, dtype=np.uint32)[None, :]).astype(np.uint32)
    s16 = (0x3C00 + np.arange(N * NG, dtype=np.uint16)).reshape(N, NG)
    z16 = (0x4000 + np.arange(N * NG, dtype=np.uint16)).reshape(N, NG)
    return P, s16, z16


def _il(w):
    """Nibble slot t <- canonical nibble 2t (t < 4) or 2(t-4)+1, bit by bit."""
    out = 0
    for t in range(8):
        src = 2 * t if t < 4 else 2 * (t - 4) + 1
        for bit in range(4):
            if (w >> (4 * src + bit)) & 1:
                out |= 1 << (4 * t + bit)
    return out


def test_interleave_hand_example():
    # nibble i of 0x76543210 is i: slots get 0,2,4,6,1,3,5,7
    assert oracle.interleave_word(0x76543210) == 0x75316420
    assert oracle.interleave_word(0xF0000000) == 0xF0000000
    assert oracle.interleave_word(0x000000F0) == 0x000F0000
    r = np.random.default_rng(4)
    for w in r.integers(0, 2 ** 32, 200, dtype=np.uint64):
        assert oracle.interleave_word(int(w)) == _il(int(w))


def _u32(buf, off):
    return int(np.frombuffer(buf[off:off + 4].tobytes(), np.uint32)[0])


def _u16(buf, off):
    return int(np.frombuffer(buf[off:off + 2].tobytes(), np.uint16)[0])


def test_layout_hand_offsets_asym():
    N, K = 3, 640                         # 5 groups: slabs of 4 and 1 group
    P, s16, z16 = _canonical(N, K)
    out = oracle.relayout(P, s16, z16, N, K, sym=False)
    full = 128 * 4 * (64 + 4)             # 34816
    assert out.size == full + 128 * 1 * 68 == oracle.layout_bytes(N, K, False)
    # row 2, group 1, word 3 -> canonical word 19 at 2*256 + 64 + 12
    assert _u32(out, 588) == _il((2 << 16) | 19)
    # its metadata: 32768 + (2*4 + 1)*4
    assert _u32(out, 32804) == int(s16[2, 1]) | (int(z16[2, 1]) << 16)
    # slab 1 (group 4), row 1, word 15 -> canonical word 79
    assert _u32(out, 34816 + 64 + 60) == _il((1 << 16) | 79)
    assert _u32(out, 34816 + 128 * 64 + 4) == int(s16[1, 4]) | (int(z16[1, 4]) << 16)
    # padding rows are zero
    assert not out[3 * 256:128 * 256].any()
    assert not out[32768 + 3 * 16:full].any()


def test_layout_hand_offsets_sym():
    N, K = 130, 1024                      # two row tiles, two full slabs
    P, s16, _ = _canonical(N, K)
    out = oracle.relayout(P, s16, None, N, K, sym=True)
    full = 128 * 4 * 66                   # 33792
    assert out.size == 2 * 2 * full
    # slab 1, row tile 1 (rows 128..255), row 129 -> r = 1, group 6 -> g = 2, word 0
    base = 1 * 2 * full + 1 * full
    assert _u32(out, base + 1 * 256 + 2 * 64) == _il((129 << 16) | (6 * 16))
    assert _u16(out, base + 128 * 256 + (1 * 4 + 2) * 2) == int(s16[129, 6])


@pytest.mark.parametrize("sym", [True, False])
def test_layout_is_a_permutation(sym):
    """Every canonical word and every scale/zero appears exactly once."""
    N, K = 200, 1408                      # ragged rows and an 11-group K
    P, s16, z16 = _canonical(N, K)
    out = oracle.relayout(P, s16, None if sym else z16, N, K, sym=sym)
    NG = K // 128
    NS, NB = (NG + 3) // 4, 2
    words, metas = [], []
    off = 0
    for s in range(NS):
        gs = min(4, NG - 4 * s)
        for b in range(NB):
            tile = out[off:off + 128 * gs * (64 + (2 if sym else 4))]
            codes = tile[:128 * gs * 64].view(np.uint32).reshape(128, gs * 16)
            meta = tile[128 * gs * 64:].view(np.uint16 if sym else np.uint32).reshape(128, gs)
            rows = min(128, N - 128 * b)
            words.append(codes[:rows].ravel())
            metas.append(meta[:rows].ravel())
            off += tile.size
    assert off == out.size
    words = np.concatenate(words)
    expect = np.array([_il(int(w)) for w in P.ravel()], np.uint32)
    assert np.array_equal(np.sort(words), np.sort(expect))
    metas = np.concatenate(metas)
    ref = s16.ravel() if sym else (s16.astype(np.uint32) | (z16.astype(np.uint32) << 16)).ravel()
    assert np.array_equal(np.sort(metas), np.sort(ref))
