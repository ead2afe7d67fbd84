"""Python binding of libvelox.so, the B200 routed block-sparse attention path.

Argument marshalling only: every function forwards device pointers, sizes
and the current CUDA stream to the C entry point of the same name declared in
include/velox.h, and raises VeloxError on a non-OK status.  All compute runs
in the library's sm_100a kernels.  Importing this package loads the library
and raises if it is missing; there is no other implementation to fall back to.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvelox.so")

VELOX_OK = 0
STATUS_NAMES = {0: "VELOX_OK", 1: "VELOX_ERR_INVALID_ARG", 2: "VELOX_ERR_UNSUPPORTED",
                3: "VELOX_ERR_WORKSPACE", 4: "VELOX_ERR_CAPACITY", 5: "VELOX_ERR_DEVICE",
                6: "VELOX_ERR_TIMEOUT", 7: "VELOX_ERR_CUDA"}
DEV_BAD_ROUTE_ID = 0x01
DEV_DUP_ROUTE_ID = 0x02
DEV_ROUTE_LEN = 0x04
DEV_NBR_OVERFLOW = 0x08
DEV_BAD_SAFEGUARD = 0x10
DEV_WAIT_TIMEOUT = 0x20
DEV_ROUTE_CAPACITY = 0x40
DEV_BAD_ROW_ORDER = 0x80
DEV_BAD_CAMERA = 0x100
DEV_BAD_CELL = 0x200
HEAD_DIM = 128
BLOCK_TOK = 128
MAX_BLOCKS = 65536
MAX_ROUTE = 4096
NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024

EXPORTS = ("velox_status_string", "velox_abi_version", "velox_gilbert_order",
           "velox_workspace_size", "velox_block_importance", "velox_route_build",
           "velox_block_sparse_attn", "velox_block_importance_noalloc",
           "velox_route_schedule", "velox_two_phase_attn", "velox_slab_overlap",
           "velox_coverage", "velox_route_audit", "velox_thw_linear_order",
           "velox_slab_table", "velox_multiwarp", "velox_multiwarp_workspace_size",
           "velox_wait_selftest")


class VeloxError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)} ({text})")
        self.status = status


class RouteParams(ctypes.Structure):
    """velox_route_params (lambda, tau, g_ref, theta_cov, theta_unc, k_cov, k_unc)."""
    _fields_ = [("lam", ctypes.c_float), ("tau", ctypes.c_float), ("g_ref", ctypes.c_float),
                ("theta_cov", ctypes.c_float), ("theta_unc", ctypes.c_float),
                ("k_cov", ctypes.c_int32), ("k_unc", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python routed_block_sparse_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.velox_status_string.restype = ctypes.c_char_p
    lib.velox_status_string.argtypes = [I]
    lib.velox_abi_version.restype = I
    lib.velox_abi_version.argtypes = []
    lib.velox_gilbert_order.restype = I
    lib.velox_gilbert_order.argtypes = [I, I, I, I, I, I, I, I, P, P, P, P, P, I, P, P]
    lib.velox_thw_linear_order.restype = I
    lib.velox_thw_linear_order.argtypes = [I, I, I, I, I, I, I, I, P, P, P, P, P, I, P, P]
    lib.velox_workspace_size.restype = I
    lib.velox_workspace_size.argtypes = [I, I, I, I, ctypes.POINTER(ctypes.c_size_t)]
    lib.velox_block_importance.restype = I
    lib.velox_block_importance.argtypes = [P, P, I, I, I, I, I, F, P, P, ctypes.c_size_t, P]
    lib.velox_block_importance_noalloc.restype = I
    lib.velox_block_importance_noalloc.argtypes = [P, P, I, I, I, I, I, F, P, P]
    lib.velox_route_build.restype = I
    lib.velox_route_build.argtypes = [P, P, P, ctypes.POINTER(RouteParams), I, I, P, P, I, P, I,
                                      I, I, I, P, P, P, I, P, ctypes.c_size_t, P, P]
    lib.velox_route_schedule.restype = I
    lib.velox_route_schedule.argtypes = [P, I, I, P, P]
    lib.velox_block_sparse_attn.restype = I
    lib.velox_block_sparse_attn.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, F, P, P, P, P]
    lib.velox_slab_overlap.restype = I
    lib.velox_slab_overlap.argtypes = [P, I, P, I, P, I, I, P, P, P]
    lib.velox_coverage.restype = I
    lib.velox_coverage.argtypes = [P, I, P, P, I, I, P, I, F, P, P, P, P]
    lib.velox_route_audit.restype = I
    lib.velox_route_audit.argtypes = [P, P, I, I, I, ctypes.POINTER(RouteParams), I, I, P, P]
    D = ctypes.c_double
    lib.velox_slab_table.restype = I
    lib.velox_slab_table.argtypes = [P, P, P, I, I, I, I, I, P, I, I, I, I, F, I, D, D, P, P, P,
                                     P]
    lib.velox_multiwarp.restype = I
    lib.velox_multiwarp.argtypes = [P, I, P, P, I, P, I, I, I, I, I, P, P, ctypes.c_size_t, P,
                                    P]
    lib.velox_multiwarp_workspace_size.restype = I
    lib.velox_multiwarp_workspace_size.argtypes = [I, I, I, I, ctypes.POINTER(ctypes.c_size_t)]
    lib.velox_two_phase_attn.restype = I
    lib.velox_two_phase_attn.argtypes = [P, P, P, P, P, P, I, P, P, I, I, I, I, I, I, F, P, P, P,
                                         P]
    lib.velox_wait_selftest.restype = I
    lib.velox_wait_selftest.argtypes = [I, P, P, P]
    return lib


_lib = _load()


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libvelox must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn: str, st: int):
    if st != VELOX_OK:
        raise VeloxError(fn, st, velox_status_string(st))


def velox_status_string(status: int) -> str:
    return _lib.velox_status_string(int(status)).decode()


def velox_abi_version() -> int:
    return int(_lib.velox_abi_version())


def velox_gilbert_order(T, H, W, n_chunks, b_tok, q_chunk=0, cache_first_block=0,
                        n_cache_blocks=0, rank_of_cell=None, cell_of_rank=None,
                        block_of_cell=None, nbr_ids=None, nbr_cnt=None, S_max=0,
                        dev_status=None, stream=None):
    st = _lib.velox_gilbert_order(T, H, W, n_chunks, b_tok, q_chunk, cache_first_block,
                                  n_cache_blocks, _ptr(rank_of_cell), _ptr(cell_of_rank),
                                  _ptr(block_of_cell), _ptr(nbr_ids), _ptr(nbr_cnt), S_max,
                                  _ptr(dev_status), _stream(stream))
    _check("velox_gilbert_order", st)


def velox_thw_linear_order(T, H, W, n_chunks, b_tok, q_chunk=0, cache_first_block=0,
                           n_cache_blocks=0, rank_of_cell=None, cell_of_rank=None,
                           block_of_cell=None, nbr_ids=None, nbr_cnt=None, S_max=0,
                           dev_status=None, stream=None):
    st = _lib.velox_thw_linear_order(T, H, W, n_chunks, b_tok, q_chunk, cache_first_block,
                                     n_cache_blocks, _ptr(rank_of_cell), _ptr(cell_of_rank),
                                     _ptr(block_of_cell), _ptr(nbr_ids), _ptr(nbr_cnt), S_max,
                                     _ptr(dev_status), _stream(stream))
    _check("velox_thw_linear_order", st)


def velox_workspace_size(H, N, M, d=HEAD_DIM) -> int:
    out = ctypes.c_size_t(0)
    _check("velox_workspace_size", _lib.velox_workspace_size(H, N, M, d, ctypes.byref(out)))
    return int(out.value)


def velox_block_importance(Q, K, H, N, M, d, b_tok, scale, p, ws, stream=None):
    st = _lib.velox_block_importance(_ptr(Q), _ptr(K), H, N, M, d, b_tok, float(scale), _ptr(p),
                                     _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check("velox_block_importance", st)


def velox_block_importance_noalloc(Q, K, H, N, M, d, b_tok, scale, p, stream=None):
    """velox_block_importance without a workspace, for callers that cannot
    allocate device memory (the library's fixed scratch array is used)."""
    st = _lib.velox_block_importance_noalloc(_ptr(Q), _ptr(K), H, N, M, d, b_tok, float(scale),
                                             _ptr(p), _stream(stream))
    _check("velox_block_importance_noalloc", st)


def velox_route_build(p, g, covered, prm: RouteParams, prev_begin, prev_count, nbr_ids,
                      nbr_cnt, S_max, ref_ids, n_ref, H, N, M, route_ids, route_len,
                      route_nbudget, R_max, ws, dev_status, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    st = _lib.velox_route_build(_ptr(p), _ptr(g), _ptr(covered), ctypes.byref(prm), prev_begin,
                                prev_count, _ptr(nbr_ids), _ptr(nbr_cnt), S_max,
                                _ptr(ref_ids) if n_ref > 0 else None, n_ref, H, N, M,
                                _ptr(route_ids), _ptr(route_len), _ptr(route_nbudget), R_max,
                                _ptr(ws), ws_bytes, _ptr(dev_status), _stream(stream))
    _check("velox_route_build", st)


def velox_route_schedule(route_len, rows, R_max, row_order, stream=None):
    st = _lib.velox_route_schedule(_ptr(route_len), rows, R_max, _ptr(row_order), _stream(stream))
    _check("velox_route_schedule", st)


def velox_block_sparse_attn(Q, K, V, route_ids, route_len, R_max, H, N, M, d, b_tok,
                            softmax_scale, O, lse=None, dev_status=None, stream=None,
                            row_order=None):
    st = _lib.velox_block_sparse_attn(_ptr(Q), _ptr(K), _ptr(V), _ptr(route_ids),
                                      _ptr(route_len), _ptr(row_order), R_max, H, N, M, d, b_tok,
                                      float(softmax_scale), _ptr(O), _ptr(lse),
                                      _ptr(dev_status), _stream(stream))
    _check("velox_block_sparse_attn", st)


def route_params(lam=2.0, tau=0.1, g_ref=0.2, theta_cov=0.9, theta_unc=0.9, k_cov=80,
                 k_unc=150) -> RouteParams:
    return RouteParams(lam, tau, g_ref, theta_cov, theta_unc, k_cov, k_unc)


def velox_two_phase_attn(Q, K, V, route_ids, route_len, R_max, K_cur, V_cur, N_cur, H, N, M, d,
                         b_tok, softmax_scale, O, lse=None, dev_status=None, stream=None,
                         row_order=None):
    st = _lib.velox_two_phase_attn(_ptr(Q), _ptr(K), _ptr(V), _ptr(route_ids), _ptr(route_len),
                                   _ptr(row_order), R_max, _ptr(K_cur), _ptr(V_cur), N_cur, H, N,
                                   M, d, b_tok, float(softmax_scale), _ptr(O), _ptr(lse),
                                   _ptr(dev_status), _stream(stream))
    _check("velox_two_phase_attn", st)


# velox_camera: 16 fp32 (fx, fy, cx, cy, R row-major, C); velox_slab: 6 fp32
# (u0, u1, v0, v1, zlo, zhi) then int32 cam, int32 valid.  Tensors of those
# layouts (camera [n][16] float32, slab [n][8] int32 view) are passed as is.
def velox_slab_overlap(cams, n_cams, q_slabs, N, h_slabs, M, grid, g, dev_status, stream=None):
    st = _lib.velox_slab_overlap(_ptr(cams), n_cams, _ptr(q_slabs), N, _ptr(h_slabs), M, grid,
                                 _ptr(g), _ptr(dev_status), _stream(stream))
    _check("velox_slab_overlap", st)


def velox_coverage(cams, n_cams, q_slabs, q_uvz, N, b, h_slabs, M, eta, rho, covered, dev_status,
                   stream=None):
    st = _lib.velox_coverage(_ptr(cams), n_cams, _ptr(q_slabs), _ptr(q_uvz), N, b, _ptr(h_slabs),
                             M, float(eta), _ptr(rho), _ptr(covered), _ptr(dev_status),
                             _stream(stream))
    _check("velox_coverage", st)


def velox_route_audit(p, g, H, N, M, prm, k_geo, k_fuse, counts, stream=None):
    st = _lib.velox_route_audit(_ptr(p), _ptr(g), H, N, M, ctypes.byref(prm), k_geo, k_fuse,
                                _ptr(counts), _stream(stream))
    _check("velox_route_audit", st)


def velox_slab_table(depth, conf, mask, F, frame_base, H, W, s, cell_of_rank, n_cells, b_tok,
                     first_block, n_blocks, c_min, n_min, p_lo, p_hi, slabs, dev_status,
                     token_uvz=None, stream=None):
    st = _lib.velox_slab_table(_ptr(depth), _ptr(conf), _ptr(mask), F, frame_base, H, W, s,
                               _ptr(cell_of_rank), n_cells, b_tok, first_block, n_blocks,
                               float(c_min), n_min, float(p_lo), float(p_hi), _ptr(slabs),
                               _ptr(token_uvz), _ptr(dev_status), _stream(stream))
    _check("velox_slab_table", st)


def velox_multiwarp_workspace_size(S, n_tgt, H, W) -> int:
    out = ctypes.c_size_t(0)
    _check("velox_multiwarp_workspace_size",
           _lib.velox_multiwarp_workspace_size(S, n_tgt, H, W, ctypes.byref(out)))
    return int(out.value)


def velox_multiwarp(cams, n_cams, src_depth, src_cam, S, tgt_cam, n_tgt, H, W, s, k_warp, zq,
                    ws, dev_status, stream=None):
    st = _lib.velox_multiwarp(_ptr(cams), n_cams, _ptr(src_depth), _ptr(src_cam), S,
                              _ptr(tgt_cam), n_tgt, H, W, s, k_warp, _ptr(zq), _ptr(ws),
                              ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream))
    _check("velox_multiwarp", st)


def velox_wait_selftest(limit_us, dev_status, elapsed_ns=None, stream=None):
    st = _lib.velox_wait_selftest(int(limit_us), _ptr(dev_status), _ptr(elapsed_ns),
                                  _stream(stream))
    _check("velox_wait_selftest", st)
