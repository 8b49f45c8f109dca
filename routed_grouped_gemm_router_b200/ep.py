"""Expert-parallel plumbing of the layer: the experts are split over the
ranks of a process group (rank r owns the contiguous block of experts
[r E_l, (r + 1) E_l), E_l = E / world) and every (token, expert) pair's row
travels to its expert's owner and back.

modelopt `moe` helpers, a2a_moe Flow: the pairs are expanded and sent to the
experts, computed there, sent back, weighted by the routing weights and
summed per token. Here:

  forward, on every rank with its own tokens:
    1. route and permute (moe_route_permute): the rows are sorted by expert,
       so the rows bound for rank d are one contiguous block;
    2. pack each row's local expert index and routing weight
       (moe_ep_pack_rows) and send rows, indices and weights to their owners
       (all-to-all);
    3. on the owner: sort the received rows by local expert (moe_permute with
       k = 1: each received row is its own "token"), run the local experts
       (moe_experts_fwd, weighted), and put the results back in arrival order
       (moe_combine with k = 1);
    4. send the results back (all-to-all, the reverse split) and sum each
       token's k rows (moe_combine).
  backward:
    1. gather dY into the same expert order (moe_permute with dY) and send
       the rows to the owners;
    2. on the owner: moe_layer_bwd_pair_dw with k = 1 gives the rows' dX in
       arrival order, the local experts' dW (complete: every row of these
       experts is here) and each row's routing-weight gradient;
    3. send dX rows and routing-weight gradients back; dX = moe_combine,
       d logits = moe_router_bwd_from_dw.

Every step of the layer runs in the CUDA library (the `ops` object, the
binding by default); this module only splits, exchanges and reassembles
rows. The split sizes are read back to the host once per forward (the
all-to-all needs them there). With gloo, CUDA tensors are exchanged through
host memory.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


class CudaOps:
    """The layer's steps as the C-ABI calls (through the binding)."""

    def __init__(self, stream=None):
        from . import binding as B
        self.B = B
        self.stream = stream

    def route_permute(self, logits, k, X):
        idx, w, probs, perm = self.B.moe_route_permute(logits, k, X, stream=self.stream)
        return idx, w, probs, perm

    def pack_rows(self, offsets, sorted_pair, topk_w, T, E, k, E_l):
        return self.B.moe_ep_pack_rows(offsets, sorted_pair, topk_w, T, E, k, E_l, stream=self.stream)

    def permute(self, ids, E, X):
        return self.B.moe_permute(ids, E, X, stream=self.stream)

    def experts_fwd(self, Xp, offsets, sorted_pair, w, T, E, k, W_gu, W_d):
        return self.B.moe_experts_fwd(Xp, offsets, sorted_pair, w, T, E, k, W_gu, W_d, save_gu=True,
                                      stream=self.stream)

    def combine(self, O, pair_pos, T, k):
        return self.B.moe_combine(O, pair_pos, T, k, stream=self.stream)

    def gather(self, idx, E, rows):
        return self.B.moe_permute(idx, E, rows, stream=self.stream)["Xp"]

    def layer_bwd_pair_dw(self, dY, Xp, gu, h, w, offsets, sorted_pair, pair_pos, T, E, k, W_gu, W_d):
        return self.B.moe_layer_bwd_pair_dw(dY, Xp, gu, h, w, offsets, sorted_pair, pair_pos, T, E, k, W_gu, W_d,
                                            stream=self.stream)

    def router_bwd_from_dw(self, dw_rows, pair_pos, probs, idx, w):
        return self.B.moe_router_bwd_from_dw(dw_rows, pair_pos, probs, idx, w, stream=self.stream)


def experts_of_rank(E: int, world: int, rank: int) -> tuple[int, int]:
    """[first, last) expert owned by `rank` when E experts are split over
    `world` ranks in contiguous blocks (E must be a multiple of world)."""
    if world <= 0 or E % world != 0 or not 0 <= rank < world:
        raise ValueError(f"{E} experts cannot be split evenly over {world} ranks (rank {rank})")
    E_l = E // world
    return rank * E_l, (rank + 1) * E_l


def _exchange(t: torch.Tensor, send_counts: list, recv_counts: list, group) -> torch.Tensor:
    """Rows (dim 0) of t, split by send_counts, go to ranks 0..world-1 in
    order; returns the rows received, grouped by source rank."""
    out = torch.empty((sum(recv_counts),) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    host = t.is_cuda and dist.get_backend(group) == "gloo"
    src = t.contiguous().cpu() if host else t.contiguous()
    dst = torch.empty(out.shape, dtype=t.dtype) if host else out
    dist.all_to_all_single(dst, src, recv_counts, send_counts, group=group)
    if host:
        out.copy_(dst)
    return out


def _exchange_counts(send_counts: list, device, group) -> list:
    dev = device if dist.get_backend(group) == "nccl" else "cpu"
    s = torch.tensor(send_counts, dtype=torch.int64, device=dev)
    r = torch.empty_like(s)
    dist.all_to_all_single(r, s, group=group)
    return r.tolist()


@dataclass
class EPState:
    T: int
    E: int
    k: int
    E_l: int
    idx: torch.Tensor
    w: torch.Tensor
    probs: torch.Tensor
    perm: dict
    send_counts: list
    recv_counts: list
    P_recv: int
    recv_w: torch.Tensor
    perm_l: dict
    h_l: torch.Tensor
    gu_l: torch.Tensor
    Y: torch.Tensor


def ep_forward(logits, X, W_gu_l, W_d_l, k: int, E: int, group=None, ops=None) -> EPState:
    """Forward of the expert-parallel layer on this rank's tokens (logits
    [T, E], X [T, H]); W_gu_l [E_l, 2I, H] / W_d_l [E_l, H, I] are this rank's
    experts. Returns the state, whose Y [T, H] is the layer's output."""
    ops = ops or CudaOps()
    world = dist.get_world_size(group)
    T = logits.shape[0]
    E_l = E // world
    experts_of_rank(E, world, dist.get_rank(group))
    idx, w, probs, perm = ops.route_permute(logits, k, X)
    offs = perm["offsets"].cpu().tolist()
    send_counts = [offs[(d + 1) * E_l] - offs[d * E_l] for d in range(world)]
    recv_counts = _exchange_counts(send_counts, X.device, group)
    local_expert, row_w = ops.pack_rows(perm["offsets"], perm["sorted_pair"], w, T, E, k, E_l)
    X_recv = _exchange(perm["Xp"], send_counts, recv_counts, group)
    ids_recv = _exchange(local_expert, send_counts, recv_counts, group)
    w_recv = _exchange(row_w, send_counts, recv_counts, group)
    P_recv = sum(recv_counts)
    perm_l = ops.permute(ids_recv.view(P_recv, 1), E_l, X_recv)
    h_l, gu_l, O_l = ops.experts_fwd(perm_l["Xp"], perm_l["offsets"], perm_l["sorted_pair"], w_recv, P_recv, E_l, 1,
                                     W_gu_l, W_d_l)
    O_back = ops.combine(O_l, perm_l["pair_pos"], P_recv, 1)
    O_sorted = _exchange(O_back, recv_counts, send_counts, group)
    Y = ops.combine(O_sorted, perm["pair_pos"], T, k)
    return EPState(T, E, k, E_l, idx, w, probs, perm, send_counts, recv_counts, P_recv, w_recv, perm_l, h_l, gu_l, Y)


def ep_backward(st: EPState, dY, W_gu_l, W_d_l, group=None, ops=None) -> dict:
    """Backward for upstream gradient dY [T, H]: dX [T, H] and d logits
    [T, E] of this rank's tokens, and dW_gu / dW_d of this rank's experts
    (summed over every rank's rows)."""
    ops = ops or CudaOps()
    dYp = ops.gather(st.idx, st.E, dY)
    dY_recv = _exchange(dYp, st.send_counts, st.recv_counts, group)
    pl = st.perm_l
    g = ops.layer_bwd_pair_dw(dY_recv, pl["Xp"], st.gu_l, st.h_l, st.recv_w, pl["offsets"], pl["sorted_pair"],
                              pl["pair_pos"], st.P_recv, st.E_l, 1, W_gu_l, W_d_l)
    dX_rows = _exchange(g["dX"], st.recv_counts, st.send_counts, group)
    dw_rows = _exchange(g["dw"], st.recv_counts, st.send_counts, group)
    dX = ops.combine(dX_rows, st.perm["pair_pos"], st.T, st.k)
    dlogits = ops.router_bwd_from_dw(dw_rows, st.perm["pair_pos"], st.probs, st.idx, st.w)
    return dict(dX=dX, dW_gu=g["dW_gu"], dW_d=g["dW_d"], dlogits=dlogits)
