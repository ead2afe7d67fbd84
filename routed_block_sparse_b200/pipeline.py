"""One routed attention layer: buffers plus the four library calls in order.

This module only allocates device buffers (through torch) and sequences the
C entry points; the arithmetic of every step runs in libvelox.so.

    layer = RoutedLayer(H, N, M, prm=route_params(), prev_begin=M - 48,
                        prev_count=48, lattice=(4, 32, 48), q_chunk=47)
    O, lse = layer.forward(Q, K, V, g, covered)

The route build is followed by velox_route_schedule (longest routes first), whose
order the attention launch follows.

Step order (Velox project page, "02 · Method", steps 03-04; digest of arXiv
2610.22311, "Method steps", step four and five): block importance -> soft
fusion and route -> block-sparse attention.  The Gilbert neighbour table is
built once per rollout shape in the constructor.
"""

from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import (BLOCK_TOK, HEAD_DIM, RouteParams, route_params, velox_block_importance,
               velox_block_sparse_attn, velox_gilbert_order, velox_route_build,
               velox_route_schedule, velox_thw_linear_order, velox_workspace_size)

DEFAULT_S_MAX = 64


class RoutedLayer:
    def __init__(self, H: int, N: int, M: int, *, prm: Optional[RouteParams] = None,
                 prev_begin: int = 0, prev_count: int = 0, lattice=None, q_chunk: int = 0,
                 cache_first_block: int = 0, S_max: int = DEFAULT_S_MAX,
                 ref_ids: Optional[torch.Tensor] = None, importance_scale: float = 1.0,
                 softmax_scale: float = 0.0, order: str = "gilbert", device="cuda"):
        self.H, self.N, self.M = H, N, M
        self.b, self.d = BLOCK_TOK, HEAD_DIM
        self.prm = prm if prm is not None else route_params()
        self.prev_begin, self.prev_count = prev_begin, prev_count
        self.importance_scale = importance_scale
        self.softmax_scale = softmax_scale
        dev = torch.device(device)
        i32 = torch.int32
        self.dev_status = torch.zeros(1, dtype=i32, device=dev)
        self.ws = torch.empty(max(velox_workspace_size(H, N, M), 256), dtype=torch.uint8,
                              device=dev)
        self.p = torch.empty(H, N, M, dtype=torch.float32, device=dev)
        self.ref_ids = ref_ids
        self.n_ref = 0 if ref_ids is None else int(ref_ids.numel())
        if lattice is not None:
            T, Hl, Wl = lattice
            n_chunks = q_chunk + 1
            assert T * Hl * Wl // self.b == N
            self.S_max = S_max
            self.nbr_ids = torch.empty(N, S_max, dtype=i32, device=dev)
            self.nbr_cnt = torch.empty(N, dtype=i32, device=dev)
            # the neighbour table of the token order the cache is stored in:
            # the global Gilbert order, or the THW-linear (raster) order the
            # pages compare it with
            if order not in ("gilbert", "thw"):
                raise ValueError(f"unknown order {order!r}")
            fn = velox_gilbert_order if order == "gilbert" else velox_thw_linear_order
            fn(T, Hl, Wl, n_chunks, self.b, q_chunk, cache_first_block, M,
               nbr_ids=self.nbr_ids, nbr_cnt=self.nbr_cnt, S_max=S_max,
               dev_status=self.dev_status)
        else:
            self.S_max = 0
            self.nbr_ids = self.nbr_cnt = None
        kmax = max(self.prm.k_cov, self.prm.k_unc, prev_count)
        self.R_max = max(1, min(M, kmax + self.S_max + self.n_ref))
        self.route_ids = torch.empty(H, N, self.R_max, dtype=i32, device=dev)
        self.route_len = torch.empty(H, N, dtype=i32, device=dev)
        self.route_nbudget = torch.empty(H, N, dtype=i32, device=dev)
        self.row_order = torch.empty(H * N, dtype=i32, device=dev)
        self.O = torch.empty(H, N * self.b, self.d, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(H, N * self.b, dtype=torch.float32, device=dev)

    # -- steps ------------------------------------------------------------
    def importance(self, Q, K, stream=None):
        velox_block_importance(Q, K, self.H, self.N, self.M, self.d, self.b,
                               self.importance_scale, self.p, self.ws, stream)
        return self.p

    def route(self, g, covered, p=None, stream=None):
        velox_route_build(self.p if p is None else p, g, covered, self.prm, self.prev_begin,
                          self.prev_count, self.nbr_ids, self.nbr_cnt, self.S_max,
                          self.ref_ids, self.n_ref, self.H, self.N, self.M, self.route_ids,
                          self.route_len, self.route_nbudget, self.R_max, self.ws,
                          self.dev_status, stream)
        velox_route_schedule(self.route_len, self.H * self.N, self.R_max, self.row_order, stream)
        return self.route_ids, self.route_len, self.route_nbudget

    def attend(self, Q, K, V, dense: bool = False, stream=None):
        velox_block_sparse_attn(Q, K, V, None if dense else self.route_ids,
                                None if dense else self.route_len, self.R_max, self.H, self.N,
                                self.M, self.d, self.b, self.softmax_scale, self.O, self.lse,
                                self.dev_status, stream,
                                row_order=None if dense else self.row_order)
        return self.O, self.lse

    def forward(self, Q, K, V, g, covered, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
        self.importance(Q, K, stream)
        self.route(g, covered, stream=stream)
        return self.attend(Q, K, V, stream=stream)

    def capture(self, Q, K, V, g, covered) -> "torch.cuda.CUDAGraph":
        """Record forward() on these tensors as a CUDA graph.

        Every call of the layer enqueues its kernels on the current stream
        and allocates nothing, so the four steps (importance, route build,
        schedule, attention: six kernels) can be captured once and replayed
        with graph.replay() for as long as the tensors stay in place (new
        values may be copied into them between replays).  One warm-up call
        before the capture sets the kernels' shared-memory attributes and
        builds the tensor maps outside it.
        """
        self.forward(Q, K, V, g, covered)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.forward(Q, K, V, g, covered)
        return graph

    def status(self) -> int:
        return int(self.dev_status.item())


def layer_for(wl, device="cuda", **kw) -> RoutedLayer:
    """A RoutedLayer sized for a synthetic workload description."""
    p = wl.params
    prm = route_params(p.lam, p.tau, p.g_ref, p.theta_cov, p.theta_unc, p.k_cov, p.k_unc)
    return RoutedLayer(wl.heads, wl.n_q_blocks, wl.n_kv_blocks, prm=prm,
                       prev_begin=wl.prev_begin, prev_count=wl.prev_count,
                       lattice=wl.lattice, q_chunk=wl.q_chunk,
                       cache_first_block=wl.cache_first_block, device=device, **kw)


def audit_metrics(counts: torch.Tensor, M: int, k_geo: int = 50, k_fuse: int = 80) -> dict:
    """Pooled ratios (sums over all rows) from the six per-row counts that
    velox_route_audit writes: R_geo, R_50, top-k_fuse recall of the
    positive-overlap blocks for the model's p and for the fused weight, and
    the fraction of the fused top-k_fuse not in the model's."""
    c = counts.reshape(-1, 6).to(torch.int64)
    rows = c.shape[0]
    t = c.sum(dim=0).tolist()
    n_pos = t[0]
    ratio = (lambda x: x / n_pos) if n_pos else (lambda x: float("nan"))
    return {"R_geo": ratio(t[1]), "R_50": t[2] / (rows * min(k_geo, M)),
            "recall_top_fuse_model": ratio(t[3]), "recall_top_fuse_fused": ratio(t[4]),
            "changed_fraction": t[5] / (rows * min(k_fuse, M)), "positive_blocks": n_pos}
