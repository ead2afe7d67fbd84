"""The C-ABI library builds, loads and exports every declared entry point.

Runs without a GPU: only host-side code of the library is exercised
(status strings, version, workspace sizing, argument validation that returns
before any CUDA call, and the device check that refuses to run without an
sm_100 device).
"""

import ctypes
import os
import re

import pytest

from conftest import ROOT, gpu_available

HEADER = os.path.join(ROOT, "include", "velox.h")


def _declared():
    text = open(HEADER).read()
    return re.findall(r"VELOX_API\s+[\w\s\*]*?\b(velox_\w+)\s*\(", text)


@pytest.fixture(scope="module")
def built():
    # load the build script by path: importing the package loads the library
    import importlib.util
    path = os.path.join(ROOT, "routed_block_sparse_b200", "build.py")
    spec = importlib.util.spec_from_file_location("velox_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


def test_header_declares_the_four_steps():
    names = _declared()
    for n in ("velox_gilbert_order", "velox_block_importance", "velox_route_build",
              "velox_block_sparse_attn", "velox_workspace_size", "velox_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(built):
    lib = ctypes.CDLL(built)
    for name in _declared():
        assert hasattr(lib, name), name
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", built], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r"\bT\s+(velox_\w+)", out))
    assert exported == set(_declared())


def test_binding_names_match_header(built):
    import routed_block_sparse_b200 as rbs
    for name in _declared():
        assert callable(getattr(rbs, name)), name
    assert set(rbs.EXPORTS) == set(_declared())


def test_status_strings_and_version(built):
    import routed_block_sparse_b200 as rbs
    assert rbs.velox_abi_version() == 104
    for s in range(8):
        assert isinstance(rbs.velox_status_string(s), str) and rbs.velox_status_string(s)
    assert rbs.velox_status_string(99) == "unknown status"


def test_workspace_size_is_host_only(built):
    import routed_block_sparse_b200 as rbs
    b = rbs.velox_workspace_size(40, 48, 2256)
    assert b >= 40 * (48 + 2256) * 128 * 4 and b % 256 == 0
    with pytest.raises(rbs.VeloxError):
        rbs.velox_workspace_size(40, 48, 2256, d=64)
    with pytest.raises(rbs.VeloxError):
        rbs.velox_workspace_size(0, 48, 2256)


def test_invalid_arguments_rejected_before_any_launch(built):
    lib = ctypes.CDLL(built)
    lib.velox_block_sparse_attn.restype = ctypes.c_int
    P = ctypes.c_void_p
    # null pointers -> VELOX_ERR_INVALID_ARG (1)
    st = lib.velox_block_sparse_attn(None, None, None, None, None, None, 0, 1, 1, 1, 128, 128,
                                     ctypes.c_float(0.0), None, None, None, None)
    assert st == 1
    fake = P(0x10000)
    # unsupported head dim -> VELOX_ERR_UNSUPPORTED (2)
    st = lib.velox_block_sparse_attn(fake, fake, fake, None, None, None, 0, 1, 1, 1, 64, 128,
                                     ctypes.c_float(0.0), fake, None, None, None)
    assert st == 2
    # R_max above the routed limit -> unsupported
    st = lib.velox_block_sparse_attn(fake, fake, fake, fake, fake, None, 5000, 1, 1, 1, 128, 128,
                                     ctypes.c_float(0.0), fake, None, fake, None)
    assert st == 2
    # a row order without a status word to report bad entries -> invalid
    st = lib.velox_block_sparse_attn(fake, fake, fake, None, None, fake, 0, 1, 1, 1, 128, 128,
                                     ctypes.c_float(0.0), fake, None, None, None)
    assert st == 1
    lib.velox_route_schedule.restype = ctypes.c_int
    assert lib.velox_route_schedule(None, 4, 10, fake, None) == 1
    assert lib.velox_route_schedule(fake, 4, 5000, fake, None) == 2
    # misaligned tensor -> invalid
    st = lib.velox_block_sparse_attn(P(0x10002), fake, fake, None, None, None, 0, 1, 1, 1, 128,
                                     128, ctypes.c_float(0.0), fake, None, None, None)
    assert st == 1
    # gilbert: W < H and W odd with H even are unsupported
    lib.velox_gilbert_order.restype = ctypes.c_int
    assert lib.velox_gilbert_order(2, 4, 3, 2, 2, 0, 0, 0, fake, None, None, None, None, 0,
                                   None, None) == 2
    assert lib.velox_gilbert_order(2, 2, 3, 2, 2, 0, 0, 0, fake, None, None, None, None, 0,
                                   None, None) == 2


def test_route_capacity_and_workspace_checks(built):
    import routed_block_sparse_b200 as rbs
    lib = ctypes.CDLL(built)
    lib.velox_route_build.restype = ctypes.c_int
    P = ctypes.c_void_p
    fake = P(0x10000)
    prm = rbs.route_params(k_cov=80, k_unc=150)
    args = [fake, fake, fake, ctypes.byref(prm), 100, 48, None, None, 0, None, 0, 40, 48, 2256,
            fake, fake, fake]
    # R_max too small for K_unc -> VELOX_ERR_CAPACITY (4)
    assert lib.velox_route_build(*args, 149, None, ctypes.c_size_t(0), fake, None) == 4
    # reserved range outside the cache -> invalid
    bad = list(args)
    bad[4] = 2250
    assert lib.velox_route_build(*bad, 200, None, ctypes.c_size_t(0), fake, None) == 1
    # K above the supported cap -> unsupported
    big = rbs.route_params(k_cov=5000, k_unc=150)
    bad = list(args)
    bad[3] = ctypes.byref(big)
    assert lib.velox_route_build(*bad, 6000, None, ctypes.c_size_t(0), fake, None) == 2


@pytest.mark.skipif(gpu_available(), reason="checks the no-device refusal")
def test_no_device_is_refused_not_emulated(built):
    lib = ctypes.CDLL(built)
    lib.velox_gilbert_order.restype = ctypes.c_int
    fake = ctypes.c_void_p(0x10000)
    # valid arguments, but no sm_100 device: VELOX_ERR_DEVICE (5), nothing runs
    assert lib.velox_gilbert_order(2, 2, 4, 2, 2, 0, 0, 0, fake, None, None, None, None, 0,
                                   None, None) == 5
    # the wait self-test: valid arguments are refused the same way
    lib.velox_wait_selftest.restype = ctypes.c_int
    assert lib.velox_wait_selftest(1000, fake, None, None) == 5


def test_wait_selftest_arguments_checked_on_the_host(built):
    lib = ctypes.CDLL(built)
    lib.velox_wait_selftest.restype = ctypes.c_int
    fake = ctypes.c_void_p(0x10000)
    assert lib.velox_wait_selftest(1000, None, None, None) == 1
    for bad in (0, -1, 2_000_001):
        assert lib.velox_wait_selftest(bad, fake, None, None) == 1


def test_clock_probe_arguments_checked_on_the_host(built):
    lib = ctypes.CDLL(built)
    lib.velox_clock_probe.restype = ctypes.c_int
    fake = ctypes.c_void_p(0x10000)
    assert lib.velox_clock_probe(None, 10, 100, None) == 1
    for n, pause in ((0, 100), (-1, 100), (1_000_001, 100), (10, -1), (10, 1_000_001)):
        assert lib.velox_clock_probe(fake, n, pause, None) == 1
    # valid arguments, no sm_100 device: refused, nothing runs
    assert lib.velox_clock_probe(fake, 10, 100, None) == 5
