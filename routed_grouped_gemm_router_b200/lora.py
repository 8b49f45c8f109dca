"""LoRA adapter formats for the stacked expert weights.

The layer takes one adapter per expert on each stacked weight, in the fused
gate|up format: A_gu [E, r, H] and B_gu [E, 2I, r] adapt W_gu [E, 2I, H] (rows
[0, I) gate, [I, 2I) up), A_d [E, r, I] and B_d [E, H, r] adapt W_d [E, H, I];
the layer then uses W + scale * B A. Adapters trained per projection (the
unfused format: one pair for the gate rows, one for the up rows) convert to
and from it exactly. Source: fused-MoE Triton project summary (sourcepulse),
Highlighted Details: LoRA on the fused expert weights, with conversion
between the fused and the unfused adapter formats.

These are one-off layout conversions of the adapter tensors (copies, no
arithmetic on their values), not steps of the layer.
"""
from __future__ import annotations

import torch


def fuse_gate_up(A_g: torch.Tensor, B_g: torch.Tensor, A_u: torch.Tensor, B_u: torch.Tensor):
    """Unfused gate / up adapters -> one fused gate|up adapter of rank r_g + r_u.

    A_g [E, r_g, H], B_g [E, I, r_g] adapt the gate rows; A_u [E, r_u, H],
    B_u [E, I, r_u] the up rows. The fused pair is A_gu = [A_g; A_u] and the
    block-diagonal B_gu = [[B_g, 0], [0, B_u]], so B_gu A_gu stacks B_g A_g
    over B_u A_u exactly (the zero blocks contribute exact zeros)."""
    E, r_g, H = A_g.shape
    r_u = A_u.shape[1]
    I = B_g.shape[1]
    if B_g.shape != (E, I, r_g) or A_u.shape != (E, r_u, H) or B_u.shape != (E, I, r_u):
        raise ValueError("adapter shapes do not match: A_g [E,r_g,H], B_g [E,I,r_g], A_u [E,r_u,H], B_u [E,I,r_u]")
    A_gu = torch.cat([A_g, A_u], dim=1).contiguous()
    B_gu = torch.zeros(E, 2 * I, r_g + r_u, dtype=B_g.dtype, device=B_g.device)
    B_gu[:, :I, :r_g] = B_g
    B_gu[:, I:, r_g:] = B_u
    return A_gu, B_gu


def unfuse_gate_up(A_gu: torch.Tensor, B_gu: torch.Tensor):
    """Fused gate|up adapter -> unfused gate and up adapters, each of rank r:
    (A_gu, B_gu[:, :I]) for the gate rows and (A_gu, B_gu[:, I:]) for the up
    rows. Exact: the rows of B_gu A_gu split the same way."""
    I2 = B_gu.shape[1]
    if I2 % 2:
        raise ValueError("B_gu must have 2I rows")
    I = I2 // 2
    return (A_gu.clone(), B_gu[:, :I].contiguous(), A_gu.clone(), B_gu[:, I:].contiguous())
