"""The five synthetic workloads of the routed attention path.

Shapes follow the chunked-generation setting of the Velox pages: one latent
chunk of T frames x H_lat x W_lat tokens forms the query side, and the KV cache
holds every earlier chunk in global Gilbert order, cut into 128-token blocks
(Velox project page, "02 · Method", "Keeping neighbours adjacent in the block
order"; digest of arXiv 2610.22311, "Method steps", step five).  Route
hyper-parameters are the ones the pages fix (tau = 0.1, g_ref = 0.2, lambda = 2,
K_cov = 80, K_unc = 150; onedev.kr summary, "How it differs").
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional

B_TOK = 128
HEAD_DIM = 128


@dataclass(frozen=True)
class RouteParams:
    lam: float = 2.0
    tau: float = 0.1
    g_ref: float = 0.2
    theta_cov: float = 0.9
    theta_unc: float = 0.9
    k_cov: int = 80
    k_unc: int = 150


@dataclass(frozen=True)
class Workload:
    """One synthetic problem instance (one layer of one attention call)."""

    name: str
    index: int                    # 1-based workload number, enters the seed
    heads: int
    n_q_blocks: int               # N
    n_kv_blocks: int              # M (history blocks in the cache)
    # geometry/value recipe
    g_kind: str = "half_zero"     # "half_zero": U[0,1] with 50% zeroed; "sparse": 10% nonzero U[0.2,1]
    cover_kind: str = "bernoulli"  # "bernoulli": p=0.5 per row; "exact70": exactly round(0.7 N) rows
    key_mean_sigma: float = 0.0   # >0: keys share a per-block mean direction ~ N(0, sigma^2 I)
    prev_count: int = 0           # reserved previous-chunk blocks = the last prev_count cache blocks
    params: RouteParams = field(default_factory=RouteParams)
    # latent lattice (None: no lattice, no neighbour safeguards)
    lattice: Optional[tuple] = None   # (T, H_lat, W_lat)
    q_chunk: int = 0
    cache_first_block: int = 0
    layer: int = 0
    d: int = HEAD_DIM
    b: int = B_TOK

    @property
    def seed(self) -> int:
        return 20261202 + 1000 * self.index + self.layer

    @property
    def n_chunks(self) -> int:
        return self.q_chunk + 1

    @property
    def prev_begin(self) -> int:
        return self.n_kv_blocks - self.prev_count

    def with_layer(self, layer: int) -> "Workload":
        return replace(self, layer=layer)


def _chunk48(M: int, index: int) -> Workload:
    T, Hl, Wl = 4, 32, 48
    per_chunk = T * Hl * Wl // B_TOK          # 48 blocks per chunk
    q_chunk = -(-M // per_chunk)              # history chunks needed to hold M blocks
    total_hist = q_chunk * per_chunk
    return Workload(
        name="chunk48" if index == 3 else f"sweep_M{M}", index=index, heads=40,
        n_q_blocks=per_chunk, n_kv_blocks=M, g_kind="half_zero",
        cover_kind="bernoulli", prev_count=min(per_chunk, M),
        params=RouteParams(), lattice=(T, Hl, Wl), q_chunk=q_chunk,
        cache_first_block=total_hist - M)


CONFIGS = {
    1: Workload(name="tiny", index=1, heads=1, n_q_blocks=2, n_kv_blocks=8,
                g_kind="half_zero", cover_kind="bernoulli", prev_count=2,
                params=RouteParams(k_cov=3, k_unc=5)),
    2: Workload(name="audit", index=2, heads=40, n_q_blocks=12, n_kv_blocks=143,
                g_kind="sparse", cover_kind="exact70", key_mean_sigma=0.5,
                prev_count=12, params=RouteParams()),
    3: _chunk48(2256, 3),
}

SWEEP_M = (64, 256, 1024, 2256, 4096)


def sweep_workload(M: int) -> Workload:
    """History-length sweep: the chunk-48 per-chunk shape with M cache blocks."""
    return _chunk48(M, 4)


def config(i: int, layer: int = 0) -> Workload:
    """Workload i (1-5); workload 5 is the chunk-48 layer with per-layer seeds
    (one Workload per layer)."""
    if i == 5:
        return replace(CONFIGS[3], index=5, name="chunk48_layers", layer=layer)
    return CONFIGS[i].with_layer(layer)


def small(heads: int, N: int, M: int, prev: int, **kw) -> Workload:
    """Ad-hoc small workload for unit and edge-case tests."""
    return Workload(name=kw.pop("name", f"small_h{heads}_n{N}_m{M}"),
                    index=kw.pop("index", 9), heads=heads, n_q_blocks=N,
                    n_kv_blocks=M, prev_count=prev, **kw)
