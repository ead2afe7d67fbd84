"""Failure detection without a GPU fault: the bounded waits end and report.

Every kernel that waits on an mbarrier bounds the wait by the device clock;
a wait that gives up sets the CTA's abort flag (ending the CTA's other
waits), and the error comes back through dev_status instead of a trap.
`velox_wait_selftest` runs that wait on barriers that nothing completes, so
the limit is reached on purpose with nothing faulting; afterwards the same
context must still compute an ordinary attention call correctly.
"""

import pytest
import torch

import routed_block_sparse_b200 as rbs
from synth.configs import small
from synth import make_inputs
from parity import assert_attention_close, attention_rows

pytestmark = pytest.mark.gpu

LIMIT_US = 100_000  # 0.1 s


def _selftest(limit_us):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    el = torch.full((2,), -1, dtype=torch.int64, device="cuda")
    rbs.velox_wait_selftest(limit_us, st, el)
    torch.cuda.synchronize()
    return int(st.item()), [int(x) for x in el.tolist()]


def test_wait_gives_up_at_its_limit_and_the_abort_flag_ends_the_others(lib):
    st, (e0, e1) = _selftest(LIMIT_US)
    assert st == rbs.DEV_WAIT_TIMEOUT
    limit_ns = LIMIT_US * 1000
    # thread 0 gives up after its limit (the clock is read every 64 tries)
    assert limit_ns <= e0 < limit_ns + 200_000_000, e0
    # the second warp's own limit is ten times longer: only the abort flag
    # can have ended its wait this early
    assert e1 < 5 * limit_ns, e1
    assert e1 >= limit_ns - 1_000_000, e1


def test_invalid_limits_are_refused_before_launch(lib):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for bad in (0, -5, 2_000_001):
        with pytest.raises(rbs.VeloxError) as e:
            rbs.velox_wait_selftest(bad, st)
        assert e.value.status == 1  # VELOX_ERR_INVALID_ARG
    with pytest.raises(rbs.VeloxError):
        rbs.velox_wait_selftest(LIMIT_US, None)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def test_context_still_computes_after_a_timeout(lib):
    st0, _ = _selftest(20_000)
    assert st0 == rbs.DEV_WAIT_TIMEOUT
    wl = small(2, 3, 9, 2)
    inp = make_inputs(wl, "cuda")
    H, N, M = wl.heads, wl.n_q_blocks, wl.n_kv_blocks
    routes = {(h, i): sorted({(3 * i + 2 * h + k) % M for k in range(4)}) for h in range(H)
              for i in range(N)}
    R_max = 4
    rid = torch.full((H, N, R_max), -1, dtype=torch.int32)
    rlen = torch.zeros(H, N, dtype=torch.int32)
    for (h, i), lst in routes.items():
        rid[h, i, :len(lst)] = torch.tensor(lst, dtype=torch.int32)
        rlen[h, i] = len(lst)
    O = torch.empty(H, N * 128, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(H, N * 128, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rbs.velox_block_sparse_attn(inp.Q, inp.K, inp.V, rid.cuda(), rlen.cuda(), R_max, H, N, M,
                                128, 128, 0.0, O, lse, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = attention_rows(inp.Q, inp.K, inp.V, sorted(routes), lambda h, i: routes[(h, i)])
    assert_attention_close(O, lse, ref)
