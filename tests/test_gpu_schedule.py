"""velox_route_schedule and the row order of the attention launch.

The schedule is a launch order: rows sorted by route length, longest first,
ties in ascending row index.  It is checked bit for bit against that
definition (Python's stable sort), and attention launched in that order must
give bitwise the same output as the natural order.
"""

import numpy as np
import pytest
import torch

import routed_block_sparse_b200 as rbs
from synth.configs import small
from synth import make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,R_max", [(1, 1), (37, 5), (1920, 214), (5000, 4096), (8192, 300),
                                        (9000, 300)])
def test_schedule_is_the_stable_longest_first_order(lib, rows, R_max):
    r = np.random.default_rng(rows)
    L = r.integers(0, R_max + 1, rows).astype(np.int32)
    if rows > 10:
        L[::7] = R_max // 2          # many ties
        L[3] = -4                     # out of range counts as 0
        L[5] = R_max + 9
    out = torch.full((rows,), -1, dtype=torch.int32, device="cuda")
    rbs.velox_route_schedule(torch.from_numpy(L).cuda(), rows, R_max, out)
    torch.cuda.synchronize()
    Lc = np.where((L < 0) | (L > R_max), 0, L)
    want = sorted(range(rows), key=lambda i: (-int(Lc[i]), i))
    assert out.cpu().tolist() == want


def _attn(inp, rid, rln, R, order=None):
    wl = inp.wl
    H, N, M = wl.heads, wl.n_q_blocks, wl.n_kv_blocks
    O = torch.full((H, N * 128, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((H, N * 128), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rbs.velox_block_sparse_attn(inp.Q, inp.K, inp.V, rid, rln, R, H, N, M, 128, 128, 0.0, O, lse,
                                st, row_order=order)
    torch.cuda.synchronize()
    return O, lse, int(st.item())


def test_row_order_changes_no_result(lib):
    H, N, M = 3, 7, 40
    inp = make_inputs(small(H, N, M, 0), "cuda")
    r = np.random.default_rng(1)
    R = 30
    ids = torch.full((H, N, R), -1, dtype=torch.int32)
    ln = torch.zeros(H, N, dtype=torch.int32)
    for h in range(H):
        for i in range(N):
            k = int(r.integers(0, R + 1))
            ids[h, i, :k] = torch.from_numpy(r.choice(M, size=k, replace=False).astype(np.int32))
            ln[h, i] = k
    rid, rln = ids.cuda(), ln.cuda()
    order = torch.empty(H * N, dtype=torch.int32, device="cuda")
    rbs.velox_route_schedule(rln, H * N, R, order)
    O0, l0, s0 = _attn(inp, rid, rln, R)
    O1, l1, s1 = _attn(inp, rid, rln, R, order)
    assert s0 == 0 and s1 == 0
    assert torch.equal(O0.view(torch.int16), O1.view(torch.int16))
    assert torch.equal(l0, l1)


def test_bad_row_order_entry_is_flagged_and_skipped(lib):
    H, N, M = 1, 4, 6
    inp = make_inputs(small(H, N, M, 0), "cuda")
    rid = torch.tensor([[[0, 1], [2, 3], [4, 5], [1, 2]]], dtype=torch.int32, device="cuda")
    rln = torch.full((H, N), 2, dtype=torch.int32, device="cuda")
    ref, _, _ = _attn(inp, rid, rln, 2)
    order = torch.tensor([3, 99, 1, 0], dtype=torch.int32, device="cuda")  # row 2 never scheduled
    O, _, st = _attn(inp, rid, rln, 2, order)
    assert st & rbs.DEV_BAD_ROW_ORDER
    for i in (0, 1, 3):
        assert torch.equal(O[0, i * 128:(i + 1) * 128].view(torch.int16),
                           ref[0, i * 128:(i + 1) * 128].view(torch.int16))
