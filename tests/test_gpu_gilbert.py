"""GPU Gilbert order and neighbour table vs the oracle: bit-exact."""

import numpy as np
import pytest
import torch

from oracle import gilbert

pytestmark = pytest.mark.gpu

ORDER_CASES = [
    # T, H, W, b, n_chunks
    (3, 3, 4, 2, 2),          # the pages' toy lattice
    (4, 32, 48, 128, 48),     # chunk-48 rollout lattice
    (4, 32, 48, 128, 87),     # the M = 4096 sweep lattice
    (3, 5, 7, 5, 3),          # odd x odd frames
    (2, 6, 10, 8, 5),
    (1, 1, 16, 4, 3),         # single-row frames
    (5, 16, 16, 64, 2),       # square power-of-two frames (Hilbert)
    (2, 9, 30, 12, 4),        # long frames (two-way splits)
]


@pytest.mark.parametrize("T,H,W,b,nc", ORDER_CASES)
def test_order_bit_exact(lib, T, H, W, b, nc):
    n = nc * T * H * W
    rank = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    cell = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    block = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    lib.velox_gilbert_order(T, H, W, nc, b, rank_of_cell=rank, cell_of_rank=cell,
                            block_of_cell=block)
    torch.cuda.synchronize()
    r_ref, c_ref, b_ref = gilbert.global_order(T, H, W, nc, b)
    assert np.array_equal(rank.cpu().numpy(), r_ref)
    assert np.array_equal(cell.cpu().numpy(), c_ref)
    assert np.array_equal(block.cpu().numpy(), b_ref)


NBR_CASES = [
    # T, H, W, b, n_chunks, q_chunk, cache_first, n_cache
    (3, 3, 4, 2, 2, 1, 0, 18),
    (3, 3, 4, 2, 3, 2, 5, 31),
    (2, 2, 4, 4, 3, 1, 0, 12),          # cache also holds later blocks
    (4, 32, 48, 128, 48, 47, 0, 2256),  # chunk-48
    (4, 32, 48, 128, 3, 2, 32, 64),     # sweep M = 64
    (2, 6, 10, 8, 5, 3, 0, 60),
]


@pytest.mark.parametrize("T,H,W,b,nc,qc,first,M", NBR_CASES)
def test_neighbours_bit_exact(lib, T, H, W, b, nc, qc, first, M):
    N = T * H * W // b
    S_max = 64
    ids = torch.full((N, S_max), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.velox_gilbert_order(T, H, W, nc, b, qc, first, M, nbr_ids=ids, nbr_cnt=cnt,
                            S_max=S_max, dev_status=st)
    torch.cuda.synchronize()
    ref = gilbert.neighbour_blocks(T, H, W, nc, b, qc, first, M)
    assert int(st.item()) == 0
    ids, cnt = ids.cpu().numpy(), cnt.cpu().numpy()
    for i in range(N):
        assert cnt[i] == len(ref[i])
        assert ids[i, :cnt[i]].tolist() == ref[i]
        assert np.all(ids[i, cnt[i]:] == -1)


def test_neighbour_overflow_is_flagged_and_cut(lib):
    T, H, W, b, nc, qc = 3, 3, 4, 2, 3, 2
    N = T * H * W // b
    S_max = 2
    ids = torch.full((N, S_max), -7, dtype=torch.int32, device="cuda")
    cnt = torch.empty(N, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.velox_gilbert_order(T, H, W, nc, b, qc, 0, 36, nbr_ids=ids, nbr_cnt=cnt, S_max=S_max,
                            dev_status=st)
    torch.cuda.synchronize()
    ref = gilbert.neighbour_blocks(T, H, W, nc, b, qc, 0, 36)
    assert any(len(r) > S_max for r in ref)
    assert int(st.item()) & lib.DEV_NBR_OVERFLOW
    for i in range(N):
        k = min(S_max, len(ref[i]))
        assert ids[i, :k].tolist() == ref[i][:k]
        assert int(cnt[i]) == k


def test_unsupported_lattices_raise(lib):
    out = torch.empty(64, dtype=torch.int32, device="cuda")
    with pytest.raises(lib.VeloxError):
        lib.velox_gilbert_order(2, 4, 3, 1, 2, rank_of_cell=out)   # W < H
    with pytest.raises(lib.VeloxError):
        lib.velox_gilbert_order(2, 2, 3, 1, 3, rank_of_cell=out)   # W odd, H even
    with pytest.raises(lib.VeloxError):
        lib.velox_gilbert_order(3, 3, 4, 1, 5, rank_of_cell=out)   # 36 % 5 != 0


THW_CASES = [
    # T, H, W, b, n_chunks
    (3, 3, 4, 2, 2),          # the pages' toy lattice
    (4, 32, 48, 128, 48),     # chunk-48 rollout lattice
    (2, 8, 5, 8, 3),          # W < H (allowed for a raster order)
]


@pytest.mark.parametrize("T,H,W,b,nc", THW_CASES)
def test_thw_order_bit_exact(lib, T, H, W, b, nc):
    n = nc * T * H * W
    rank = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    block = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    lib.velox_thw_linear_order(T, H, W, nc, b, rank_of_cell=rank, block_of_cell=block)
    torch.cuda.synchronize()
    r_ref, _, b_ref = gilbert.thw_linear_order(T, H, W, nc, b)
    assert np.array_equal(rank.cpu().numpy(), r_ref)
    assert np.array_equal(block.cpu().numpy(), b_ref)


@pytest.mark.parametrize("T,H,W,b,nc,qc,first,M", [
    (3, 3, 4, 2, 2, 1, 0, 18),
    (4, 32, 48, 128, 48, 47, 0, 2256),  # chunk-48
    (2, 8, 5, 8, 3, 1, 2, 12),
    (1, 96, 96, 128, 3, 2, 0, 144),     # frame above the shared-memory table size
])
def test_thw_neighbours_bit_exact(lib, T, H, W, b, nc, qc, first, M):
    N = T * H * W // b
    S_max = 64
    ids = torch.full((N, S_max), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.velox_thw_linear_order(T, H, W, nc, b, qc, first, M, nbr_ids=ids, nbr_cnt=cnt,
                               S_max=S_max, dev_status=st)
    torch.cuda.synchronize()
    ref = gilbert.neighbour_blocks(T, H, W, nc, b, qc, first, M, layout="thw")
    assert int(st.item()) == 0
    c = cnt.cpu().numpy()
    got = ids.cpu().numpy()
    for i in range(N):
        assert c[i] == len(ref[i])
        assert got[i, :c[i]].tolist() == ref[i]
        assert np.all(got[i, c[i]:] == -1)


def _random_lattices(seed, n):
    """Seeded supported lattices: W >= H, not (W odd and H even), b a
    divisor of T H W (>= 4 keeps the oracle's neighbour search quick)."""
    r = np.random.default_rng(seed)
    out = []
    while len(out) < n:
        T = int(r.integers(1, 4))
        H = int(r.integers(1, 13))
        W = int(r.integers(H, 25))
        if W % 2 == 1 and H % 2 == 0:
            continue
        cells = T * H * W
        divs = [d for d in range(4, min(cells, 256) + 1) if cells % d == 0]
        if not divs:
            continue
        b = int(r.choice(divs))
        nc = int(r.integers(2, 5))
        out.append((T, H, W, b, nc))
    return out


@pytest.mark.parametrize("T,H,W,b,nc", _random_lattices(20261203, 20))
def test_random_lattices_order_and_neighbours_bit_exact(lib, T, H, W, b, nc):
    n = nc * T * H * W
    rank = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    cell = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    block = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    N = T * H * W // b
    qc, M = nc - 1, (nc - 1) * N
    S_max = 256
    ids = torch.full((N, S_max), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.velox_gilbert_order(T, H, W, nc, b, qc, 0, M, rank_of_cell=rank, cell_of_rank=cell,
                            block_of_cell=block, nbr_ids=ids, nbr_cnt=cnt, S_max=S_max,
                            dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    r_ref, c_ref, b_ref = gilbert.global_order(T, H, W, nc, b)
    assert np.array_equal(rank.cpu().numpy(), r_ref)
    assert np.array_equal(cell.cpu().numpy(), c_ref)
    assert np.array_equal(block.cpu().numpy(), b_ref)
    ref = gilbert.neighbour_blocks(T, H, W, nc, b, qc, 0, M)
    ids, cnt = ids.cpu().numpy(), cnt.cpu().numpy()
    for i in range(N):
        assert cnt[i] == len(ref[i]) and ids[i, :cnt[i]].tolist() == ref[i]
