"""Seeded input draws for one Workload.

Q, K, V are bf16 draws of N(0, 1) (rounded to nearest even from fp32 by torch),
head-major and contiguous: Q is [H][N*b][d], K and V are [H][M*b][d], tokens in
global Gilbert order.  With ``key_mean_sigma > 0`` every key block r of head h
gets a shared offset mu_{h,r} ~ N(0, sigma^2 I) before rounding, so that the
mean keys differ between blocks.

g is [N][M] fp32 and covered is [N] uint8.  They are drawn on the CPU from their
own seeded generator so that they are identical whichever device holds Q/K/V.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

from .configs import Workload


@dataclass
class Inputs:
    wl: Workload
    Q: torch.Tensor        # [H][N*b][d] bf16
    K: torch.Tensor        # [H][M*b][d] bf16
    V: torch.Tensor        # [H][M*b][d] bf16
    g: torch.Tensor        # [N][M] fp32
    covered: torch.Tensor  # [N] uint8
    ref_ids: torch.Tensor  # [n_ref] int32 (empty in every config)


def _geometry(wl: Workload):
    gen = torch.Generator(device="cpu").manual_seed(wl.seed * 7 + 1)
    N, M = wl.n_q_blocks, wl.n_kv_blocks
    if wl.g_kind == "half_zero":
        g = torch.rand(N, M, generator=gen, dtype=torch.float32)
        zero = torch.rand(N, M, generator=gen) < 0.5
        g[zero] = 0.0
    elif wl.g_kind == "sparse":
        u = torch.rand(N, M, generator=gen, dtype=torch.float32)
        keep = torch.rand(N, M, generator=gen) < 0.1
        g = torch.where(keep, 0.2 + 0.8 * u, torch.zeros_like(u))
    elif wl.g_kind == "zero":
        g = torch.zeros(N, M, dtype=torch.float32)
    else:
        raise ValueError(f"unknown g_kind {wl.g_kind}")
    if wl.cover_kind == "bernoulli":
        covered = (torch.rand(N, generator=gen) < 0.5).to(torch.uint8)
    elif wl.cover_kind == "exact70":
        covered = torch.zeros(N, dtype=torch.uint8)
        covered[torch.randperm(N, generator=gen)[: round(0.7 * N)]] = 1
    elif wl.cover_kind == "all":
        covered = torch.ones(N, dtype=torch.uint8)
    elif wl.cover_kind == "none":
        covered = torch.zeros(N, dtype=torch.uint8)
    else:
        raise ValueError(f"unknown cover_kind {wl.cover_kind}")
    return g.contiguous(), covered.contiguous()


def make_inputs(wl: Workload, device="cpu", out: Optional[Inputs] = None,
                heads: Optional[tuple] = None) -> Inputs:
    """Draw the inputs of ``wl`` on ``device``; reuse ``out``'s buffers if given.

    ``heads=(h0, h1)`` keeps only heads h0..h1-1 of Q, K and V: the values are
    those heads of the full draw (the whole layer is drawn, then cut), so the
    shares of several ranks put together are the single-rank inputs.  The
    returned workload then has h1 - h0 heads.
    """
    if heads is not None:
        from dataclasses import replace
        h0, h1 = heads
        if not (0 <= h0 < h1 <= wl.heads):
            raise ValueError(f"head range {heads} outside 0..{wl.heads}")
        full = make_inputs(wl, device)
        cut = lambda t: t[h0:h1].clone()
        return Inputs(wl=replace(wl, heads=h1 - h0), Q=cut(full.Q), K=cut(full.K),
                      V=cut(full.V), g=full.g, covered=full.covered, ref_ids=full.ref_ids)
    device = torch.device(device)
    H, N, M, b, d = wl.heads, wl.n_q_blocks, wl.n_kv_blocks, wl.b, wl.d
    gen = torch.Generator(device=device).manual_seed(wl.seed)
    bf = torch.bfloat16
    if out is None:
        Q = torch.empty(H, N * b, d, dtype=bf, device=device)
        K = torch.empty(H, M * b, d, dtype=bf, device=device)
        V = torch.empty(H, M * b, d, dtype=bf, device=device)
    else:
        Q, K, V = out.Q, out.K, out.V
    Q.normal_(generator=gen)
    V.normal_(generator=gen)
    if wl.key_mean_sigma > 0:
        mu = torch.randn(H, M, 1, d, generator=gen, device=device) * wl.key_mean_sigma
        noise = torch.randn(H, M, b, d, generator=gen, device=device)
        K.copy_((mu + noise).reshape(H, M * b, d))
        del mu, noise
    else:
        K.normal_(generator=gen)
    g, covered = _geometry(wl)
    ref = torch.zeros(0, dtype=torch.int32)
    return Inputs(wl=wl, Q=Q, K=K, V=V, g=g.to(device), covered=covered.to(device),
                  ref_ids=ref.to(device))


def make_current(wl: Workload, device="cpu", n_blocks: Optional[int] = None):
    """K and V of the chunk being generated, [H][n*b][d] bf16 ~ N(0, 1) with
    n = n_blocks (default: the workload's N query blocks): the second phase
    of two-phase attention (its own seed, disjoint from Q/K/V)."""
    device = torch.device(device)
    gen = torch.Generator(device=device).manual_seed(wl.seed * 7 + 5)
    n = wl.n_q_blocks if n_blocks is None else n_blocks
    shape = (wl.heads, n * wl.b, wl.d)
    Kc = torch.empty(shape, dtype=torch.bfloat16, device=device).normal_(generator=gen)
    Vc = torch.empty(shape, dtype=torch.bfloat16, device=device).normal_(generator=gen)
    return Kc, Vc
