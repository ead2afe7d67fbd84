"""The Python binding's marshalling checks (no GPU needed for these).

The C ABI takes raw device pointers and cannot see a tensor's device, dtype
or size; the binding checks them before the call, so a host tensor, a
wrong dtype or a tensor smaller than the sizes given never reaches a kernel.
The dtype and size checks on CUDA tensors are in test_gpu_binding_checks.py.
"""

import pytest
import torch

import routed_block_sparse_b200 as rbs


def test_host_tensors_are_refused_before_the_call():
    x = torch.zeros(16)
    with pytest.raises(ValueError, match="CUDA device"):
        rbs.velox_block_sparse_attn(x, x, x, None, None, 0, 1, 1, 1, 128, 128, 0.0, x)
    with pytest.raises(ValueError, match="CUDA device"):
        rbs.velox_route_schedule(torch.zeros(4, dtype=torch.int32), 4, 10,
                                 torch.zeros(4, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA device"):
        rbs.velox_wait_selftest(1000, torch.zeros(1, dtype=torch.int32))


def test_non_tensors_are_refused():
    with pytest.raises(TypeError):
        rbs.velox_wait_selftest(1000, [0])


def test_element_counts_follow_the_sizes():
    assert rbs._n(40, 48, 128, 128) == 40 * 48 * 128 * 128
    # a size the library refuses itself: no count check on the Python side
    assert rbs._n(40, 0, 128) == 0 and rbs._n(-1, 5) == 0


def test_null_optional_arguments_reach_the_library():
    # dev_status is required: NULL goes through and the library refuses it
    with pytest.raises(rbs.VeloxError) as e:
        rbs.velox_wait_selftest(1000, None, stream=0)
    assert e.value.status == 1
