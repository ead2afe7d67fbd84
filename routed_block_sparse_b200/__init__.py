"""Python binding of libvelox.so, the B200 routed block-sparse attention path.

Argument marshalling only: every function forwards device pointers, sizes
and the current CUDA stream to the C entry point of the same name declared in
include/velox.h, and raises VeloxError on a non-OK status.  Before the call it
checks what the C ABI cannot see on a raw pointer (each tensor on a CUDA
device, of the expected dtype, contiguous, with at least the elements the
sizes imply) and raises ValueError or TypeError otherwise.  All compute runs
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
           "velox_wait_selftest", "velox_clock_probe")


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
    lib.velox_clock_probe.restype = I
    lib.velox_clock_probe.argtypes = [P, I, I, P]
    return lib


_lib = _load()


BF16 = (torch.bfloat16,)
F32 = (torch.float32,)
I32 = (torch.int32,)
U8 = (torch.uint8,)
W32 = (torch.int32, torch.float32)  # camera / slab records: 4-byte words


def _n(*factors) -> int:
    """Element count the sizes call for; 0 (no check) when a size is not
    positive, which the library itself refuses."""
    out = 1
    for f in factors:
        if f <= 0:
            return 0
        out *= int(f)
    return out


def _arg(t: Optional[torch.Tensor], name: str, dtypes=None, numel: int = 0):
    """Device pointer of `t` (None stays NULL) after the checks the C ABI
    cannot make on a raw pointer: a torch tensor on a CUDA device, of one of
    `dtypes`, contiguous, and holding at least `numel` elements."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.device.type != "cuda":
        raise ValueError(f"{name}: tensors passed to libvelox must be on a CUDA device "
                         f"(got {t.device})")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected one of {list(dtypes)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: tensors passed to libvelox must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name}: {t.numel()} elements, the sizes given need {numel}")
    return ctypes.c_void_p(t.data_ptr())


def _ptr(t: Optional[torch.Tensor], name: str = "workspace"):
    """Device pointer of a buffer of any dtype (workspaces: the library checks
    their byte count itself)."""
    return _arg(t, name)


def _nbytes(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.numel() * t.element_size()


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


def _order_args(T, H, W, n_chunks, b_tok, rank_of_cell, cell_of_rank, block_of_cell, nbr_ids,
                nbr_cnt, S_max):
    cells = _n(n_chunks, T, H, W)
    qb = _n(T, H, W) // b_tok if b_tok > 0 else 0  # query blocks of one chunk
    return (_arg(rank_of_cell, "rank_of_cell", I32, cells),
            _arg(cell_of_rank, "cell_of_rank", I32, cells),
            _arg(block_of_cell, "block_of_cell", I32, cells),
            _arg(nbr_ids, "nbr_ids", I32, _n(qb, S_max)), _arg(nbr_cnt, "nbr_cnt", I32, qb))


def velox_gilbert_order(T, H, W, n_chunks, b_tok, q_chunk=0, cache_first_block=0,
                        n_cache_blocks=0, rank_of_cell=None, cell_of_rank=None,
                        block_of_cell=None, nbr_ids=None, nbr_cnt=None, S_max=0,
                        dev_status=None, stream=None):
    st = _lib.velox_gilbert_order(T, H, W, n_chunks, b_tok, q_chunk, cache_first_block,
                                  n_cache_blocks, *_order_args(T, H, W, n_chunks, b_tok,
                                                               rank_of_cell, cell_of_rank,
                                                               block_of_cell, nbr_ids, nbr_cnt,
                                                               S_max), S_max,
                                  _arg(dev_status, "dev_status", I32, 1), _stream(stream))
    _check("velox_gilbert_order", st)


def velox_thw_linear_order(T, H, W, n_chunks, b_tok, q_chunk=0, cache_first_block=0,
                           n_cache_blocks=0, rank_of_cell=None, cell_of_rank=None,
                           block_of_cell=None, nbr_ids=None, nbr_cnt=None, S_max=0,
                           dev_status=None, stream=None):
    st = _lib.velox_thw_linear_order(T, H, W, n_chunks, b_tok, q_chunk, cache_first_block,
                                     n_cache_blocks, *_order_args(T, H, W, n_chunks, b_tok,
                                                                  rank_of_cell, cell_of_rank,
                                                                  block_of_cell, nbr_ids,
                                                                  nbr_cnt, S_max), S_max,
                                     _arg(dev_status, "dev_status", I32, 1), _stream(stream))
    _check("velox_thw_linear_order", st)


def velox_workspace_size(H, N, M, d=HEAD_DIM) -> int:
    out = ctypes.c_size_t(0)
    _check("velox_workspace_size", _lib.velox_workspace_size(H, N, M, d, ctypes.byref(out)))
    return int(out.value)


def velox_block_importance(Q, K, H, N, M, d, b_tok, scale, p, ws, stream=None):
    st = _lib.velox_block_importance(_arg(Q, "Q", BF16, _n(H, N, b_tok, d)),
                                     _arg(K, "K", BF16, _n(H, M, b_tok, d)), H, N, M, d, b_tok,
                                     float(scale), _arg(p, "p", F32, _n(H, N, M)), _ptr(ws),
                                     _nbytes(ws), _stream(stream))
    _check("velox_block_importance", st)


def velox_block_importance_noalloc(Q, K, H, N, M, d, b_tok, scale, p, stream=None):
    """velox_block_importance without a workspace, for callers that cannot
    allocate device memory (the library's fixed scratch array is used)."""
    st = _lib.velox_block_importance_noalloc(_arg(Q, "Q", BF16, _n(H, N, b_tok, d)),
                                             _arg(K, "K", BF16, _n(H, M, b_tok, d)), H, N, M, d,
                                             b_tok, float(scale), _arg(p, "p", F32, _n(H, N, M)),
                                             _stream(stream))
    _check("velox_block_importance_noalloc", st)


def velox_route_build(p, g, covered, prm: RouteParams, prev_begin, prev_count, nbr_ids,
                      nbr_cnt, S_max, ref_ids, n_ref, H, N, M, route_ids, route_len,
                      route_nbudget, R_max, ws, dev_status, stream=None):
    st = _lib.velox_route_build(_arg(p, "p", F32, _n(H, N, M)), _arg(g, "g", F32, _n(N, M)),
                                _arg(covered, "covered", U8, _n(N)), ctypes.byref(prm),
                                prev_begin, prev_count,
                                _arg(nbr_ids, "nbr_ids", I32, _n(N, S_max)),
                                _arg(nbr_cnt, "nbr_cnt", I32, _n(N)), S_max,
                                _arg(ref_ids, "ref_ids", I32, _n(n_ref)) if n_ref > 0 else None,
                                n_ref, H, N, M,
                                _arg(route_ids, "route_ids", I32, _n(H, N, R_max)),
                                _arg(route_len, "route_len", I32, _n(H, N)),
                                _arg(route_nbudget, "route_nbudget", I32, _n(H, N)), R_max,
                                _ptr(ws), _nbytes(ws), _arg(dev_status, "dev_status", I32, 1),
                                _stream(stream))
    _check("velox_route_build", st)


def velox_route_schedule(route_len, rows, R_max, row_order, stream=None):
    st = _lib.velox_route_schedule(_arg(route_len, "route_len", I32, _n(rows)), rows, R_max,
                                   _arg(row_order, "row_order", I32, _n(rows)), _stream(stream))
    _check("velox_route_schedule", st)


def _attn_args(Q, K, V, route_ids, route_len, row_order, R_max, H, N, M, d, b_tok):
    return (_arg(Q, "Q", BF16, _n(H, N, b_tok, d)), _arg(K, "K", BF16, _n(H, M, b_tok, d)),
            _arg(V, "V", BF16, _n(H, M, b_tok, d)),
            _arg(route_ids, "route_ids", I32, _n(H, N, R_max)),
            _arg(route_len, "route_len", I32, _n(H, N)),
            _arg(row_order, "row_order", I32, _n(H, N)))


def velox_block_sparse_attn(Q, K, V, route_ids, route_len, R_max, H, N, M, d, b_tok,
                            softmax_scale, O, lse=None, dev_status=None, stream=None,
                            row_order=None):
    st = _lib.velox_block_sparse_attn(*_attn_args(Q, K, V, route_ids, route_len, row_order,
                                                  R_max, H, N, M, d, b_tok), R_max, H, N, M, d,
                                      b_tok, float(softmax_scale),
                                      _arg(O, "O", BF16, _n(H, N, b_tok, d)),
                                      _arg(lse, "lse", F32, _n(H, N, b_tok)),
                                      _arg(dev_status, "dev_status", I32, 1), _stream(stream))
    _check("velox_block_sparse_attn", st)


def route_params(lam=2.0, tau=0.1, g_ref=0.2, theta_cov=0.9, theta_unc=0.9, k_cov=80,
                 k_unc=150) -> RouteParams:
    return RouteParams(lam, tau, g_ref, theta_cov, theta_unc, k_cov, k_unc)


def velox_two_phase_attn(Q, K, V, route_ids, route_len, R_max, K_cur, V_cur, N_cur, H, N, M, d,
                         b_tok, softmax_scale, O, lse=None, dev_status=None, stream=None,
                         row_order=None):
    st = _lib.velox_two_phase_attn(*_attn_args(Q, K, V, route_ids, route_len, row_order, R_max,
                                               H, N, M, d, b_tok), R_max,
                                   _arg(K_cur, "K_cur", BF16, _n(H, N_cur, b_tok, d)),
                                   _arg(V_cur, "V_cur", BF16, _n(H, N_cur, b_tok, d)), N_cur, H,
                                   N, M, d, b_tok, float(softmax_scale),
                                   _arg(O, "O", BF16, _n(H, N, b_tok, d)),
                                   _arg(lse, "lse", F32, _n(H, N, b_tok)),
                                   _arg(dev_status, "dev_status", I32, 1), _stream(stream))
    _check("velox_two_phase_attn", st)


# velox_camera: 16 fp32 (fx, fy, cx, cy, R row-major, C); velox_slab: 6 fp32
# (u0, u1, v0, v1, zlo, zhi) then int32 cam, int32 valid.  Tensors of those
# layouts (camera [n][16] float32, slab [n][8] int32 view) are passed as is.
def velox_slab_overlap(cams, n_cams, q_slabs, N, h_slabs, M, grid, g, dev_status, stream=None):
    st = _lib.velox_slab_overlap(_arg(cams, "cams", W32, _n(n_cams, 16)), n_cams,
                                 _arg(q_slabs, "q_slabs", W32, _n(N, 8)), N,
                                 _arg(h_slabs, "h_slabs", W32, _n(M, 8)), M, grid,
                                 _arg(g, "g", F32, _n(N, M)),
                                 _arg(dev_status, "dev_status", I32, 1), _stream(stream))
    _check("velox_slab_overlap", st)


def velox_coverage(cams, n_cams, q_slabs, q_uvz, N, b, h_slabs, M, eta, rho, covered, dev_status,
                   stream=None):
    st = _lib.velox_coverage(_arg(cams, "cams", W32, _n(n_cams, 16)), n_cams,
                             _arg(q_slabs, "q_slabs", W32, _n(N, 8)),
                             _arg(q_uvz, "q_uvz", F32, _n(N, b, 3)), N, b,
                             _arg(h_slabs, "h_slabs", W32, _n(M, 8)), M, float(eta),
                             _arg(rho, "rho", F32, _n(N)), _arg(covered, "covered", U8, _n(N)),
                             _arg(dev_status, "dev_status", I32, 1), _stream(stream))
    _check("velox_coverage", st)


def velox_route_audit(p, g, H, N, M, prm, k_geo, k_fuse, counts, stream=None):
    st = _lib.velox_route_audit(_arg(p, "p", F32, _n(H, N, M)), _arg(g, "g", F32, _n(N, M)), H,
                                N, M, ctypes.byref(prm), k_geo, k_fuse,
                                _arg(counts, "counts", I32, _n(H, N, 6)), _stream(stream))
    _check("velox_route_audit", st)


def velox_slab_table(depth, conf, mask, F, frame_base, H, W, s, cell_of_rank, n_cells, b_tok,
                     first_block, n_blocks, c_min, n_min, p_lo, p_hi, slabs, dev_status,
                     token_uvz=None, stream=None):
    samples = _n(F, H, s, W, s)
    st = _lib.velox_slab_table(_arg(depth, "depth", F32, samples),
                               _arg(conf, "conf", F32, samples), _arg(mask, "mask", U8, samples),
                               F, frame_base, H, W, s,
                               _arg(cell_of_rank, "cell_of_rank", I32, _n(n_cells)), n_cells,
                               b_tok, first_block, n_blocks, float(c_min), n_min, float(p_lo),
                               float(p_hi), _arg(slabs, "slabs", W32, _n(n_blocks, 8)),
                               _arg(token_uvz, "token_uvz", F32, _n(n_blocks, b_tok, 3)),
                               _arg(dev_status, "dev_status", I32, 1), _stream(stream))
    _check("velox_slab_table", st)


def velox_multiwarp_workspace_size(S, n_tgt, H, W) -> int:
    out = ctypes.c_size_t(0)
    _check("velox_multiwarp_workspace_size",
           _lib.velox_multiwarp_workspace_size(S, n_tgt, H, W, ctypes.byref(out)))
    return int(out.value)


def velox_multiwarp(cams, n_cams, src_depth, src_cam, S, tgt_cam, n_tgt, H, W, s, k_warp, zq,
                    ws, dev_status, stream=None):
    st = _lib.velox_multiwarp(_arg(cams, "cams", W32, _n(n_cams, 16)), n_cams,
                              _arg(src_depth, "src_depth", F32, _n(S, H, s, W, s)),
                              _arg(src_cam, "src_cam", I32, _n(S)), S,
                              _arg(tgt_cam, "tgt_cam", I32, _n(n_tgt)), n_tgt, H, W, s, k_warp,
                              _arg(zq, "zq", F32, _n(n_tgt, H, W)), _ptr(ws), _nbytes(ws),
                              _arg(dev_status, "dev_status", I32, 1), _stream(stream))
    _check("velox_multiwarp", st)


def velox_clock_probe(samples, n, pause_ns=2000, stream=None):
    st = _lib.velox_clock_probe(_arg(samples, "samples", (torch.int64,), _n(n, 2)), int(n),
                                int(pause_ns), _stream(stream))
    _check("velox_clock_probe", st)


def velox_wait_selftest(limit_us, dev_status, elapsed_ns=None, stream=None):
    st = _lib.velox_wait_selftest(int(limit_us), _arg(dev_status, "dev_status", I32, 1),
                                  _arg(elapsed_ns, "elapsed_ns", (torch.int64,), 2),
                                  _stream(stream))
    _check("velox_wait_selftest", st)
