"""The GEMV's split of its tiles over the persistent grid (host arithmetic,
no GPU): every tile has exactly one owner team, and no team without tiles
sits among the owners of a row tile, so every split-K sum is finished.

The split is the library's own (wq_debug_gemv_split); the owner rule it is
checked with is the kernel's: team t of T owns tiles [t*tiles/T,
(t+1)*tiles/T), and a row tile's last piece waits for one piece from each
team between the owners of its first and last tile."""
import numpy as np
import pytest

from post_weight_quantization_wq_b200 import _binding as abi


def _owner(u, T, G):
    return ((u + 1) * G + T - 1) // T - 1


def _check_split(M, N, K, awq, sms, per_sm):
    st, tiles, teams, grid = abi.wq_debug_gemv_split(M, N, K, awq, sms, per_sm)
    assert st == abi.WQ_OK
    NB, NS = -(-N // 128), -(-(K // 128) // 4)
    assert tiles == NB * NS
    assert 1 <= grid <= sms * per_sm
    G = grid * teams
    assert G <= tiles + 1 or grid == 1
    runs = [(t * tiles // G, (t + 1) * tiles // G) for t in range(G)]
    assert runs[0][0] == 0 and runs[-1][1] == tiles
    assert all(a[1] == b[0] for a, b in zip(runs, runs[1:]))
    nonempty = np.array([b > a for a, b in runs])
    for b in range(NB):
        first, last = _owner(b * NS, tiles, G), _owner(b * NS + NS - 1, tiles, G)
        assert runs[first][0] <= b * NS < runs[first][1]
        assert runs[last][0] <= b * NS + NS - 1 < runs[last][1]
        assert nonempty[first:last + 1].all(), (M, N, K, b, first, last)


@pytest.mark.parametrize("M,awq", [(1, 0), (1, 1), (2, 0), (3, 0), (4, 1), (8, 0)])
def test_split_leaves_no_idle_team_inside_a_row_tile(M, awq):
    rng = np.random.default_rng(M * 10 + awq)
    shapes = [(1, 2048), (64, 1664), (100, 3200), (128, 3584), (600, 1024), (8192, 28672),
              (28672, 8192), (1, 128), (129, 11008)]
    shapes += [(int(n), 128 * int(k)) for n, k in zip(rng.integers(1, 3000, 300),
                                                       rng.integers(1, 120, 300))]
    for N, K in shapes:
        for sms, per_sm in ((148, 1), (148, 2), (7, 1)):
            _check_split(M, N, K, awq, sms, per_sm)


def test_split_of_the_headline_linear():
    """8192 x 28672: 3,584 tiles.  At M = 1 (CUDA cores) one CTA per SM of
    148 with two teams each (296 teams, 12 or 13 tiles each); at M = 2..8 the
    tensor-core kernel, one team per CTA (24 or 25 tiles each), or two teams
    again when forced onto the CUDA cores."""
    st, tiles, teams, grid = abi.wq_debug_gemv_split(1, 8192, 28672, 0, 148, 1)
    assert (st, tiles, teams, grid) == (abi.WQ_OK, 3584, 2, 148)
    for M, awq in ((2, 0), (4, 0), (3, 1), (8, 0), (6, 1)):
        st, tiles, teams, grid = abi.wq_debug_gemv_split(M, 8192, 28672, awq, 148, 1)
        assert (st, tiles, teams, grid) == (abi.WQ_OK, 3584, 1, 148)
    abi.wq_debug_gemv_force_cuda_cores(1)
    try:
        st, tiles, teams, grid = abi.wq_debug_gemv_split(2, 8192, 28672, 0, 148, 1)
    finally:
        abi.wq_debug_gemv_force_cuda_cores(0)
    assert (st, tiles, teams, grid) == (abi.WQ_OK, 3584, 2, 148)


@pytest.mark.parametrize("forced", [0, 1])
def test_split_invariants_on_both_kernels(forced):
    abi.wq_debug_gemv_force_cuda_cores(forced)
    try:
        for M in (1, 2, 4):
            for N, K in ((8192, 28672), (28672, 8192), (128, 28672), (1, 512), (300, 1536)):
                for sms, per_sm in ((148, 1), (7, 1)):
                    _check_split(M, N, K, 0, sms, per_sm)
    finally:
        abi.wq_debug_gemv_force_cuda_cores(0)


@pytest.mark.parametrize("args", [(0, 1, 128, 0, 148, 1), (9, 1, 128, 0, 148, 1),
                                  (1, 0, 128, 0, 148, 1), (1, 1, 100, 0, 148, 1),
                                  (1, 1, 128, 0, 0, 1), (1, 1, 128, 0, 148, 0)])
def test_split_validation(args):
    assert abi.wq_debug_gemv_split(*args)[0] == abi.WQ_ERR_INVALID_ARG
