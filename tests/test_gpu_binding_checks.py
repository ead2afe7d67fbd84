"""The binding's dtype and size checks on CUDA tensors: a wrong dtype or a
buffer smaller than the sizes given is refused before anything is launched
(the outputs and dev_status stay untouched)."""

import pytest
import torch

import routed_block_sparse_b200 as rbs

pytestmark = pytest.mark.gpu

H, N, M, R = 2, 3, 5, 4


def _bufs():
    bf = dict(dtype=torch.bfloat16, device="cuda")
    Q = torch.randn(H, N * 128, 128, **bf)
    K = torch.randn(H, M * 128, 128, **bf)
    V = torch.randn(H, M * 128, 128, **bf)
    rid = torch.tensor([0, 1, 2, 3] * (H * N), dtype=torch.int32, device="cuda").view(H, N, R)
    rlen = torch.full((H, N), R, dtype=torch.int32, device="cuda")
    O = torch.full((H, N * 128, 128), float("nan"), **bf)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    return Q, K, V, rid, rlen, O, st


def _untouched(O, st):
    torch.cuda.synchronize()
    assert torch.isnan(O.float()).all() and int(st.item()) == 0


def test_wrong_dtype_is_refused(lib):
    Q, K, V, rid, rlen, O, st = _bufs()
    with pytest.raises(ValueError, match="dtype"):
        rbs.velox_block_sparse_attn(Q.float(), K, V, rid, rlen, R, H, N, M, 128, 128, 0.0, O,
                                    dev_status=st)
    with pytest.raises(ValueError, match="dtype"):
        rbs.velox_block_sparse_attn(Q, K, V, rid.long(), rlen, R, H, N, M, 128, 128, 0.0, O,
                                    dev_status=st)
    _untouched(O, st)


def test_undersized_buffers_are_refused(lib):
    Q, K, V, rid, rlen, O, st = _bufs()
    with pytest.raises(ValueError, match="elements"):
        rbs.velox_block_sparse_attn(Q, K[:, :-128].contiguous(), V, rid, rlen, R, H, N, M, 128, 128, 0.0, O,
                                    dev_status=st)
    with pytest.raises(ValueError, match="elements"):  # R_max larger than the id tensor
        rbs.velox_block_sparse_attn(Q, K, V, rid, rlen, R + 1, H, N, M, 128, 128, 0.0, O,
                                    dev_status=st)
    with pytest.raises(ValueError, match="elements"):
        rbs.velox_block_sparse_attn(Q, K, V, rid, rlen, R, H, N, M, 128, 128, 0.0, O[:1],
                                    dev_status=st)
    with pytest.raises(ValueError, match="CUDA device"):
        rbs.velox_block_sparse_attn(Q, K, V, rid, rlen, R, H, N, M, 128, 128, 0.0, O,
                                    dev_status=st.cpu())
    _untouched(O, st)
    # the same call with the right tensors runs
    rbs.velox_block_sparse_attn(Q, K, V, rid, rlen, R, H, N, M, 128, 128, 0.0, O, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and torch.isfinite(O.float()).all()
