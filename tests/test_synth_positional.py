"""The positional Q/K recipe (synth.positional): seeded, order-independent
token values, and inner products that fall off with lattice distance."""

import torch

from synth.positional import cell_positions, positional_qk


def test_cell_positions_decode():
    H, W = 3, 5
    cells = torch.tensor([0, 4, 5, 14, 15, 2 * 15 + 7])
    pos = cell_positions(cells, H, W)
    assert pos.tolist() == [[0, 0, 0], [0, 0, 4], [0, 1, 0], [0, 2, 4], [1, 0, 0], [2, 1, 2]]


def test_same_token_same_values_under_any_order():
    H, W, F = 4, 6, 3
    n = F * H * W
    cells = torch.arange(n, dtype=torch.int32)
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(3)).to(torch.int32)
    Q1, K1 = positional_qk(cells[:8], cells, 2, H, W, n, d=16, seed=5)
    Q2, K2 = positional_qk(perm[:8], perm, 2, H, W, n, d=16, seed=5)
    # row j of K2 is the token of cell perm[j], i.e. row perm[j] of K1
    assert torch.equal(K2, K1[:, perm.long()])
    # likewise for Q: every query cell gets the values it has in any order
    Q_all, _ = positional_qk(cells, cells, 2, H, W, n, d=16, seed=5)
    assert torch.equal(Q2, Q_all[:, perm[:8].long()])
    assert torch.equal(Q1, Q_all[:, :8])
    assert Q1.dtype == torch.bfloat16 and Q1.shape == (2, 8, 16) and K1.shape == (2, n, 16)
    # seeded
    Q3, K3 = positional_qk(cells[:8], cells, 2, H, W, n, d=16, seed=5)
    assert torch.equal(Q3, Q1) and torch.equal(K3, K1)


def test_inner_product_falls_with_distance():
    # one frame, a 1 x 64 strip: mean q . k over pairs at distance 0 is far
    # above the mean at distance >= 4 length scales
    H, W = 1, 64
    n = H * W
    cells = torch.arange(n, dtype=torch.int32)
    Q, K = positional_qk(cells, cells, 8, H, W, n, d=128, seed=11, amp=4.0, ell_xy=4.0)
    Qf, Kf = Q.float(), K.float()
    dots = torch.einsum("hid,hjd->hij", Qf, Kf).mean(0)
    idx = torch.arange(n)
    dist = (idx[:, None] - idx[None, :]).abs()
    near = dots[dist == 0].mean()
    far = dots[dist >= 16].mean()
    assert near > 10.0 and abs(far) < 2.0, (near, far)
