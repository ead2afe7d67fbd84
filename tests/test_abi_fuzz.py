"""Host-side argument validation under random and extreme sizes (no GPU).

Every entry point validates its sizes on the host before it touches the
device.  These properties drive that validation with random integers,
extreme ones included (powers of two up to 2^31 - 1, negatives, zero), and
fake device pointers:

* a call never crashes and returns one of the documented statuses;
* whenever a call gets past validation (on a machine without an sm_100
  device it then returns VELOX_ERR_DEVICE and launches nothing), the sizes
  satisfy every documented limit, checked here with exact integers, so no
  size product can have overflowed inside the check.

Skipped where a GPU is present: there a call that passes validation would
launch a kernel on the fake pointers.
"""

import ctypes

import pytest
from hypothesis import given, settings, strategies as st

from conftest import gpu_available

pytestmark = pytest.mark.skipif(gpu_available(), reason="needs a machine without a GPU")

OK_DEVICE = 5  # VELOX_ERR_DEVICE: validation passed, no usable device
STATUSES = {1, 2, 3, 4, 5}
I32 = 2**31 - 1
FAKE = ctypes.c_void_p(0x10000)

sizes = st.one_of(
    st.integers(-3, 300),
    st.sampled_from([2**15, 2**16, 2**20, 2**24, 2**30, I32, -(2**31)]),
    st.integers(-(2**31), I32),
)


@pytest.fixture(scope="module")
def lib():
    import routed_block_sparse_b200 as rbs
    lib = ctypes.CDLL(rbs.LIB_PATH)
    I, P, F, D, Z = ctypes.c_int, ctypes.c_void_p, ctypes.c_float, ctypes.c_double, ctypes.c_size_t
    lib.velox_gilbert_order.restype = I
    lib.velox_gilbert_order.argtypes = [I, I, I, I, I, I, I, I, P, P, P, P, P, I, P, P]
    lib.velox_block_importance.restype = I
    lib.velox_block_importance.argtypes = [P, P, I, I, I, I, I, F, P, P, Z, P]
    lib.velox_block_sparse_attn.restype = I
    lib.velox_block_sparse_attn.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, F, P, P, P, P]
    lib.velox_slab_table.restype = I
    lib.velox_slab_table.argtypes = [P, P, P, I, I, I, I, I, P, I, I, I, I, F, I, D, D, P, P, P,
                                     P]
    lib.velox_multiwarp.restype = I
    lib.velox_multiwarp.argtypes = [P, I, P, P, I, P, I, I, I, I, I, P, P, Z, P, P]
    return lib


@settings(max_examples=400, deadline=None)
@given(T=sizes, H=sizes, W=sizes, n_chunks=sizes, b=sizes)
def test_gilbert_order_sizes(lib, T, H, W, n_chunks, b):
    s = lib.velox_gilbert_order(T, H, W, n_chunks, b, 0, 0, 0, FAKE, None, None, None, None, 0,
                                None, None)
    assert s in STATUSES
    if s == OK_DEVICE:
        assert min(T, H, W, n_chunks, b) > 0
        assert n_chunks * T * H * W <= I32
        assert (T * H * W) % b == 0 and b <= 1024
        assert W >= H and not (W % 2 == 1 and H % 2 == 0)


@settings(max_examples=300, deadline=None)
@given(H=sizes, N=sizes, M=sizes)
def test_importance_sizes(lib, H, N, M):
    s = lib.velox_block_importance(FAKE, FAKE, H, N, M, 128, 128, 1.0, FAKE, FAKE, 2**62, None)
    assert s in STATUSES
    if s == OK_DEVICE:
        assert min(H, N, M) > 0 and M <= 65536
        assert H * M * 128 <= I32 and H * N * 128 <= I32


@settings(max_examples=300, deadline=None)
@given(H=sizes, N=sizes, M=sizes)
def test_dense_attention_sizes(lib, H, N, M):
    s = lib.velox_block_sparse_attn(FAKE, FAKE, FAKE, None, None, None, 0, H, N, M, 128, 128,
                                    0.0, FAKE, None, None, None)
    assert s in STATUSES
    if s == OK_DEVICE:
        assert min(H, N, M) > 0 and M <= 65536
        assert M * 128 <= I32 and N * 128 <= I32 and H * N <= I32


@settings(max_examples=400, deadline=None)
@given(F=sizes, H=sizes, W=sizes, s=sizes, b=sizes, n_cells=sizes, first=sizes, n=sizes)
def test_slab_table_sizes(lib, F, H, W, s, b, n_cells, first, n):
    st_ = lib.velox_slab_table(FAKE, None, None, F, 0, H, W, s, FAKE, n_cells, b, first, n, 0.5,
                               1, 0.1, 0.9, FAKE, None, FAKE, None)
    assert st_ in STATUSES
    if st_ == OK_DEVICE:
        assert min(F, H, W, s, b, n, n_cells) > 0 and first >= 0
        assert (first + n) * b <= n_cells
        assert (H * W) % b == 0
        assert b * s * s <= 16384
        assert F * H * W * s * s <= I32


@settings(max_examples=300, deadline=None)
@given(H=sizes, W=sizes, s=sizes, S=sizes, n_tgt=sizes)
def test_multiwarp_sizes(lib, H, W, s, S, n_tgt):
    st_ = lib.velox_multiwarp(FAKE, 4, FAKE, FAKE, S, FAKE, n_tgt, H, W, s, 2, FAKE, FAKE, 2**62,
                              FAKE, None)
    assert st_ in STATUSES
    if st_ == OK_DEVICE:
        assert min(H, W, s, S, n_tgt) > 0
        assert H * W * s * s <= 32768 and H * W <= 8192
        assert S <= 65535 and n_tgt <= 65535


def test_the_overflowing_products_are_refused(lib):
    # products that wrap a 64-bit integer: 2^16 per factor, and s close to 2^31
    assert lib.velox_gilbert_order(2**16, 2**16, 2**16, 2**16, 128, 0, 0, 0, FAKE, None, None,
                                   None, None, 0, None, None) == 2
    assert lib.velox_slab_table(FAKE, None, None, 1, 0, 4, 1, I32, FAKE, I32, 4, 0, 1, 0.5, 1,
                                0.1, 0.9, FAKE, None, FAKE, None) == 2
    assert lib.velox_multiwarp(FAKE, 4, FAKE, FAKE, 1, FAKE, 1, 2**16, 2**16, 2**16, 2, FAKE,
                               FAKE, 2**62, FAKE, None) == 2


class _Prm(ctypes.Structure):
    _fields_ = [("lam", ctypes.c_float), ("tau", ctypes.c_float), ("g_ref", ctypes.c_float),
                ("theta_cov", ctypes.c_float), ("theta_unc", ctypes.c_float),
                ("k_cov", ctypes.c_int32), ("k_unc", ctypes.c_int32)]


@settings(max_examples=400, deadline=None)
@given(H=sizes, N=sizes, M=sizes, R_max=sizes, k_cov=sizes, k_unc=sizes, prev_begin=sizes,
       prev_count=sizes, S_max=sizes)
def test_route_build_sizes(lib, H, N, M, R_max, k_cov, k_unc, prev_begin, prev_count, S_max):
    f = lib.velox_route_build
    f.restype = ctypes.c_int
    prm = _Prm(2.0, 0.1, 0.2, 0.9, 0.9, k_cov, k_unc)
    nbr = FAKE if S_max > 0 else None
    s = f(FAKE, FAKE, FAKE, ctypes.byref(prm), prev_begin, prev_count, nbr, nbr, S_max, None, 0,
          H, N, M, FAKE, FAKE, FAKE, R_max, FAKE, ctypes.c_size_t(2**62), FAKE, None)
    assert s in STATUSES
    if s == OK_DEVICE:
        assert min(H, N, M) > 0 and M <= 65536 and H * N <= I32 // 2
        assert 0 <= prev_begin and 0 <= prev_count and prev_begin + prev_count <= M
        assert 0 <= k_cov <= 4096 and 0 <= k_unc <= 4096 and S_max >= 0
        assert R_max >= min(M, max(k_cov, k_unc, prev_count) + max(S_max, 0)) and R_max > 0


@settings(max_examples=300, deadline=None)
@given(N=sizes, M=sizes, grid=sizes, n_cams=sizes, b=sizes)
def test_geometry_sizes(lib, N, M, grid, n_cams, b):
    f = lib.velox_slab_overlap
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                  ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    s = f(FAKE, n_cams, FAKE, N, FAKE, M, grid, FAKE, FAKE, None)
    assert s in STATUSES
    if s == OK_DEVICE:
        assert min(N, M, grid, n_cams) > 0 and grid <= 32 and N <= 65535 and N * M <= I32
    c = lib.velox_coverage
    c.restype = ctypes.c_int
    c.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                  ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    s = c(FAKE, n_cams, FAKE, FAKE, N, b, FAKE, M, 0.9, FAKE, FAKE, FAKE, None)
    assert s in STATUSES
    if s == OK_DEVICE:
        assert min(N, M, b, n_cams) > 0 and b <= 128 and 4 * N <= I32


@settings(max_examples=300, deadline=None)
@given(H=sizes, N=sizes, M=sizes, k_geo=sizes, k_fuse=sizes)
def test_audit_sizes(lib, H, N, M, k_geo, k_fuse):
    f = lib.velox_route_audit
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    prm = _Prm(2.0, 0.1, 0.2, 0.9, 0.9, 80, 150)
    s = f(FAKE, FAKE, H, N, M, ctypes.byref(prm), k_geo, k_fuse, FAKE, None)
    assert s in STATUSES
    if s == OK_DEVICE:
        assert min(H, N, M) > 0 and k_geo >= 1 and k_fuse >= 1
        assert M <= 4096 and H * N <= I32
