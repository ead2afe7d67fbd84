"""Q and K whose inner products follow the distance between token positions.

The random Q/K of ``make_inputs`` give a block importance that knows nothing
of where a block is, so every token order routes alike.  For comparing token
orders (the global Gilbert order against the THW-linear raster) the inputs
here give each token a position (frame f, row y, column x) and make q . k
larger the closer two tokens are in space and time, as the attention of a
video model over its own latent frames would be.

Per head, d random Fourier features of the position stand in for a
positional code: frequencies w_c ~ N(0, diag(1/l_t^2, 1/l_xy^2, 1/l_xy^2)),
phases b_c ~ U[0, 2 pi), phi_c(p) = sqrt(2/d) cos(w_c . p + b_c), so that
phi(p) . phi(p') approximates exp(-|(p - p') / l|^2 / 2) (random features
for a Gaussian kernel: Rahimi and Recht, "Random Features for Large-Scale
Kernel Machines", NIPS 2007).  A token at position p gets

    q = amp * phi(p) + n_q,      k = amp * phi(p) + n_k,

with n ~ N(0, I_d) drawn per token (indexed by its lattice cell, not by its
row), so a token has the same values under every order: only the row it
occupies in Q or K changes.  Everything is seeded; nothing of the method's
arithmetic is here.
"""

from __future__ import annotations

import math

import torch


def cell_positions(cells: torch.Tensor, H: int, W: int) -> torch.Tensor:
    """(f, y, x) of lattice cells c = (f * H + y) * W + x, as an [n, 3] fp32
    tensor on the cells' device."""
    c = cells.to(torch.int64)
    f = c // (H * W)
    y = (c // W) % H
    x = c % W
    return torch.stack([f, y, x], dim=1).to(torch.float32)


def positional_qk(q_cells: torch.Tensor, k_cells: torch.Tensor, heads: int, H: int, W: int,
                  n_cells: int, d: int = 128, seed: int = 20261204, amp: float = 2.0,
                  ell_xy: float = 6.0, ell_t: float = 48.0):
    """Q [heads][len(q_cells)][d] and K [heads][len(k_cells)][d] bf16 on the
    cells' device: row j of Q holds the token of lattice cell q_cells[j] (row
    j of K that of k_cells[j]).  n_cells bounds the cell ids (the per-token
    noise is drawn for every cell of the lattice, in cell order)."""
    dev = q_cells.device
    gen = torch.Generator(device=dev).manual_seed(seed)
    pq = cell_positions(q_cells, H, W)
    pk = cell_positions(k_cells, H, W)
    scale = torch.tensor([1.0 / ell_t, 1.0 / ell_xy, 1.0 / ell_xy], device=dev)
    Q = torch.empty(heads, pq.shape[0], d, dtype=torch.bfloat16, device=dev)
    K = torch.empty(heads, pk.shape[0], d, dtype=torch.bfloat16, device=dev)
    norm = math.sqrt(2.0 / d)
    for h in range(heads):
        w = torch.randn(d, 3, generator=gen, device=dev) * scale
        b = torch.rand(d, generator=gen, device=dev) * (2.0 * math.pi)
        # per-cell noise for q and k, drawn in cell order, picked by row
        nq = torch.randn(n_cells, d, generator=gen, device=dev)
        Q[h] = (amp * norm * torch.cos(pq @ w.T + b) + nq[q_cells.long()]).to(torch.bfloat16)
        del nq
        nk = torch.randn(n_cells, d, generator=gen, device=dev)
        K[h] = (amp * norm * torch.cos(pk @ w.T + b) + nk[k_cells.long()]).to(torch.bfloat16)
        del nk
    return Q, K
