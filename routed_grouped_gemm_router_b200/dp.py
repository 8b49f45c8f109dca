"""Data-parallel plumbing of the expert layer: token shards and the
weight-gradient exchange.

The layer partitions over tokens. Routing, the permutation, the expert MLPs,
the combine and every per-token gradient (dX, d logits) depend only on the
token's own row, so each rank runs the layer on its own tokens with
replicated weights and the forward needs no exchange. The weight gradients
are sums over tokens (dW_e = sum over the expert's rows), so the gradient of
the whole batch is the sum of the ranks' gradients: one all-reduce (sum) of
dW_gu, dW_d (and the router's dW_r) per backward, or a reduce-scatter when
each rank keeps only its shard of the optimiser state. This is the
data-parallel (DDP) option that the fused-MoE Triton project summary
(sourcepulse), Limitations & Caveats, mentions; expert parallelism's two
all-to-alls are not used.

Nothing here computes the layer: it slices token ranges, lays the weight
gradients out in one flat buffer so that one collective covers them all, and
issues the collective through torch.distributed (NCCL on GPUs, gloo on CPUs).
"""
from __future__ import annotations

import torch


def token_shard(T: int, world: int, rank: int) -> tuple[int, int]:
    """[start, stop) of rank's tokens when T tokens are split over `world`
    ranks: contiguous, sizes differ by at most one, earlier ranks larger."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    base, extra = divmod(T, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def flat_views(shapes: dict, dtype, device=None) -> tuple[torch.Tensor, dict]:
    """One contiguous buffer cut into row-major views of the given shapes,
    in the order given. Every view starts on a 16-byte boundary when each
    shape's element count times the element size is a multiple of 16."""
    sizes = {n: int(torch.Size(sh).numel()) for n, sh in shapes.items()}
    flat = torch.empty(sum(sizes.values()), dtype=dtype, device=device)
    views, at = {}, 0
    for n, sh in shapes.items():
        views[n] = flat[at:at + sizes[n]].view(*sh)
        at += sizes[n]
    return flat, views


def flat_weight_grads(E: int, H: int, I: int, dtype=torch.bfloat16, device=None,
                      router: bool = False) -> tuple[torch.Tensor, dict]:
    """One contiguous buffer holding dW_gu [E, 2I, H], dW_d [E, H, I] and, with
    router=True, dW_r [E, H] (always fp32: the router is an fp32 Linear, so its
    gradient gets a buffer of its own). Returns (flat, views); the views are
    what the layer's backward writes (every view starts on a 16-byte boundary
    since H and I are multiples of 8). dW_r, when asked for, is returned in
    views but lives outside `flat`."""
    flat, views = flat_views({"dW_gu": (E, 2 * I, H), "dW_d": (E, H, I)}, dtype, device)
    if router:
        views["dW_r"] = torch.empty(E, H, dtype=torch.float32, device=device)
    return flat, views


def sync_weight_grads(flat: torch.Tensor, extra: list[torch.Tensor] | None = None, op: str = "allreduce",
                      group=None) -> torch.Tensor | None:
    """Sums the ranks' weight gradients.

    op="allreduce": every rank ends with the whole batch's gradient in `flat`
    (and in each tensor of `extra`). op="reduce_scatter": rank r ends with
    its 1/world slice of the summed `flat` (returned, rank-contiguous slices,
    `flat` padded with zeros to a multiple of world); tensors in `extra` are
    all-reduced. Collectives are issued on the current stream in a fixed
    order, the same on every rank."""
    import torch.distributed as dist

    if op not in ("allreduce", "reduce_scatter"):
        raise ValueError(f"unknown gradient exchange {op!r}")
    out = None
    if op == "allreduce":
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    else:
        world = dist.get_world_size(group)
        n = flat.numel()
        per = -(-n // world)
        src = flat
        if per * world != n:
            src = torch.zeros(per * world, dtype=flat.dtype, device=flat.device)
            src[:n].copy_(flat)
        out = torch.empty(per, dtype=flat.dtype, device=flat.device)
        dist.reduce_scatter_tensor(out, src, op=dist.ReduceOp.SUM, group=group)
    for t in extra or []:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return out
