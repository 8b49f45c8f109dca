"""The whole expert layer as a sequence of the C-ABI calls.

``forward`` runs moe_route_permute (moe_route and moe_permute in one call)
-> moe_experts_fwd -> moe_combine and returns Y plus the saved state; ``backward`` runs moe_layer_bwd. With
gather=True the permute makes no Xp copy and the GEMMs read X and dY rows by
token index (moe_experts_fwd_x / moe_layer_bwd_x): no Xp / dYp buffers
(2 x T*k*H bf16 less memory), but the row-gather loads make those GEMMs
slower, so the default keeps the permuted copies.
``forward_from_x`` / ``backward_to_x`` also run the router Linear
(moe_router_fwd in place of moe_route; moe_router_bwd after moe_layer_bwd,
adding the router's share to dX and giving dW_r). ``forward_lora`` /
``backward_lora`` run the layer with LoRA adapters on the stacked expert
weights (moe_experts_fwd_lora / moe_layer_bwd_lora). All buffers are torch
CUDA tensors; nothing here does arithmetic.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import binding as B


@dataclass
class LayerState:
    T: int
    E: int
    k: int
    topk_idx: torch.Tensor
    topk_w: torch.Tensor
    probs: torch.Tensor
    perm: dict
    h: torch.Tensor
    gu: torch.Tensor | None
    O: torch.Tensor
    Y: torch.Tensor
    logits: torch.Tensor | None = None
    X: torch.Tensor | None = None  # token-order input, kept for the gather-fused backward
    lora: dict | None = None       # adapters {A_gu, B_gu, A_d, B_d, scale} of a forward_lora
    Z_gu: torch.Tensor | None = None  # scale * Xp A_gu^T [P, r]
    Z_d: torch.Tensor | None = None   # scale * h A_d^T [P, r]


def forward(logits: torch.Tensor, X: torch.Tensor, W_gu: torch.Tensor, W_d: torch.Tensor, k: int,
            save_gu: bool = True, bufs: dict | None = None, stream=None, gather: bool = False) -> LayerState:
    """Y = combine(experts(permute(X, route(logits)))). ``bufs`` may hold
    preallocated outputs/workspaces (keys as in the returned state)."""
    b = bufs or {}
    T, E = logits.shape
    idx, w, probs, perm = B.moe_route_permute(logits, k, None if gather else X, b.get("topk_idx"), b.get("topk_w"),
                                              b.get("probs"), out=b.get("perm"), ws=b.get("route_perm_ws"),
                                              stream=stream)
    return _experts_forward(T, E, k, idx, w, probs, X, W_gu, W_d, save_gu, b, stream, gather, perm=perm)


def forward_from_x(X: torch.Tensor, W_r: torch.Tensor, W_gu: torch.Tensor, W_d: torch.Tensor, k: int,
                   save_gu: bool = True, bufs: dict | None = None, stream=None, gather: bool = False) -> LayerState:
    """As ``forward``, with the logits computed on the GPU from the fp32
    router weight W_r [E, H] (moe_router_fwd)."""
    b = bufs or {}
    T, E = X.shape[0], W_r.shape[0]
    out = {n: b[n] for n in ("logits", "topk_idx", "topk_w", "probs") if b.get(n) is not None}
    r = B.moe_router_fwd(X, W_r, k, out=out, ws=b.get("router_ws"), stream=stream)
    st = _experts_forward(T, E, k, r["topk_idx"], r["topk_w"], r["probs"], X, W_gu, W_d, save_gu, b, stream,
                          gather)
    st.logits = r["logits"]
    return st


def _experts_forward(T, E, k, idx, w, probs, X, W_gu, W_d, save_gu, b, stream, gather, perm=None) -> LayerState:
    if perm is None:
        perm = B.moe_permute(idx, E, None if gather else X, out=b.get("perm"), ws=b.get("perm_ws"), stream=stream)
    h, gu, O = B.moe_experts_fwd(X if gather else perm["Xp"], perm["offsets"], perm["sorted_pair"], w, T, E, k,
                                 W_gu, W_d, h=b.get("h"), gu_save=b.get("gu"), O=b.get("O"), save_gu=save_gu,
                                 stream=stream, gather=gather)
    Y = B.moe_combine(O, perm["pair_pos"], T, k, Y=b.get("Y"), stream=stream)
    return LayerState(T, E, k, idx, w, probs, perm, h, gu, O, Y, X=X if gather else None)


def forward_lora(logits: torch.Tensor, X: torch.Tensor, W_gu: torch.Tensor, W_d: torch.Tensor, k: int, lora: dict,
                 save_gu: bool = True, bufs: dict | None = None, stream=None) -> LayerState:
    """``forward`` with the adapted weights W + scale B A (lora = {A_gu [E,r,H],
    B_gu [E,2I,r], A_d [E,r,I], B_d [E,H,r] bf16, scale})."""
    b = bufs or {}
    T, E = logits.shape
    idx, w, probs, perm = B.moe_route_permute(logits, k, X, b.get("topk_idx"), b.get("topk_w"), b.get("probs"),
                                              out=b.get("perm"), ws=b.get("route_perm_ws"), stream=stream)
    h, gu, O, Z_gu, Z_d = B.moe_experts_fwd_lora(perm["Xp"], perm["offsets"], perm["sorted_pair"], w, T, E, k, W_gu,
                                                 W_d, lora, h=b.get("h"), gu_save=b.get("gu"), O=b.get("O"),
                                                 Z_gu=b.get("Z_gu"), Z_d=b.get("Z_d"), save_gu=save_gu,
                                                 stream=stream)
    Y = B.moe_combine(O, perm["pair_pos"], T, k, Y=b.get("Y"), stream=stream)
    return LayerState(T, E, k, idx, w, probs, perm, h, gu, O, Y, lora=lora, Z_gu=Z_gu, Z_d=Z_d)


def backward_lora(st: LayerState, dY: torch.Tensor, W_gu: torch.Tensor, W_d: torch.Tensor, bufs: dict | None = None,
                  stream=None, accumulate: bool = False, base_grads: bool = False) -> dict:
    """dX, dlogits and the fp32 adapter gradients dA_gu, dB_gu, dA_d, dB_d
    (accumulate=True adds them to the buffers in bufs["grads"]); the base
    weights are frozen unless base_grads=True."""
    b = bufs or {}
    p = st.perm
    return B.moe_layer_bwd_lora(dY, p["Xp"], st.gu, st.h, st.probs, st.topk_idx, st.topk_w, p["offsets"],
                                p["sorted_pair"], p["pair_pos"], st.T, st.E, st.k, W_gu, W_d, st.lora, st.Z_gu,
                                st.Z_d, out=b.get("grads"), ws=b.get("bwd_ws"), stream=stream,
                                accumulate=accumulate, base_grads=base_grads)


def backward(st: LayerState, dY: torch.Tensor, W_gu: torch.Tensor, W_d: torch.Tensor, bufs: dict | None = None,
             stream=None, accumulate: bool = False) -> dict:
    """dX, dW_gu, dW_d, dlogits for upstream gradient dY. The weight
    gradients are bf16, or fp32 when the buffers in bufs["grads"] are fp32
    (``allocate(..., dw_f32=True)``); accumulate=True adds to those fp32
    buffers instead of overwriting them."""
    b = bufs or {}
    p = st.perm
    gather = st.X is not None
    grads = b.get("grads")
    dw_dtype = grads["dW_gu"].dtype if grads and "dW_gu" in grads else torch.bfloat16
    return B.moe_layer_bwd(dY, st.X if gather else p["Xp"], st.gu, st.h, st.probs, st.topk_idx, st.topk_w,
                           p["offsets"], p["sorted_pair"], p["pair_pos"], st.T, st.E, st.k, W_gu, W_d,
                           out=grads, ws=b.get("bwd_ws"), stream=stream, gather=gather, dw_dtype=dw_dtype,
                           accumulate=accumulate)


def backward_to_x(st: LayerState, dY: torch.Tensor, X: torch.Tensor, W_r: torch.Tensor, W_gu: torch.Tensor,
                  W_d: torch.Tensor, bufs: dict | None = None, stream=None, accumulate: bool = False) -> dict:
    """``backward`` plus the router Linear's: dX gains dlogits W_r (in place)
    and the result holds dW_r = dlogits^T X."""
    b = bufs or {}
    g = backward(st, dY, W_gu, W_d, bufs=b, stream=stream, accumulate=accumulate)
    dW_r, _ = B.moe_router_bwd(g["dlogits"], X, W_r, dX=g["dX"], dW_r=b.get("dW_r"), ws=b.get("router_ws"),
                               stream=stream)
    g["dW_r"] = dW_r
    return g


def allocate(T: int, E: int, k: int, H: int, I: int, device, save_gu: bool = True, router: bool = False,
             gather: bool = False, dw_f32: bool = False, lora_r: int = 0) -> dict:
    """Every output and workspace of one forward+backward, allocated once;
    dw_f32: fp32 weight-gradient buffers; lora_r > 0: the buffers of
    forward_lora / backward_lora with adapters of rank lora_r (frozen base
    weights: no dW buffers)."""
    P = T * k
    bf = torch.bfloat16
    dwt = torch.float32 if dw_f32 else bf
    lib = B.lib()
    d = dict(
        topk_idx=torch.empty(T, k, dtype=torch.int32, device=device),
        topk_w=torch.empty(T, k, dtype=torch.float32, device=device),
        probs=torch.empty(T, E, dtype=torch.float32, device=device),
        perm=dict(counts=torch.empty(E, dtype=torch.int32, device=device),
                  offsets=torch.empty(E + 1, dtype=torch.int32, device=device),
                  sorted_pair=torch.empty(P, dtype=torch.int32, device=device),
                  pair_pos=torch.empty(P, dtype=torch.int32, device=device)),
        perm_ws=torch.empty(max(lib.moe_permute_workspace_bytes(T, E, k), 1), dtype=torch.uint8, device=device),
        route_perm_ws=torch.empty(max(lib.moe_route_permute_workspace_bytes(T, E, k), 1), dtype=torch.uint8,
                                  device=device),
        h=torch.empty(P, I, dtype=bf, device=device),
        gu=torch.empty(P, 2 * I, dtype=bf, device=device) if save_gu else None,
        O=torch.empty(P, H, dtype=bf, device=device),
        Y=torch.empty(T, H, dtype=bf, device=device),
        grads=dict(dX=torch.empty(T, H, dtype=bf, device=device),
                   dW_gu=torch.empty(E, 2 * I, H, dtype=dwt, device=device),
                   dW_d=torch.empty(E, H, I, dtype=dwt, device=device),
                   dlogits=torch.empty(T, E, dtype=torch.float32, device=device)),
        bwd_ws=torch.empty(max((lib.moe_layer_bwd_x_workspace_bytes if gather else lib.moe_layer_bwd_workspace_bytes)(
            T, E, k, H, I, 0 if save_gu else 1), 1), dtype=torch.uint8, device=device),
    )
    if not gather:
        d["perm"]["Xp"] = torch.empty(P, H, dtype=bf, device=device)
    if lora_r > 0:
        r = lora_r
        f32 = torch.float32
        d["Z_gu"] = torch.empty(P, r, dtype=bf, device=device)
        d["Z_d"] = torch.empty(P, r, dtype=bf, device=device)
        g = d["grads"]
        del g["dW_gu"], g["dW_d"]
        g.update(dA_gu=torch.empty(E, r, H, dtype=f32, device=device),
                 dB_gu=torch.empty(E, 2 * I, r, dtype=f32, device=device),
                 dA_d=torch.empty(E, r, I, dtype=f32, device=device),
                 dB_d=torch.empty(E, H, r, dtype=f32, device=device))
        d["bwd_ws"] = torch.empty(max(lib.moe_layer_bwd_lora_workspace_bytes(T, E, k, H, I, r, 0 if save_gu else 1),
                                      1), dtype=torch.uint8, device=device)
    if router:
        d["logits"] = torch.empty(T, E, dtype=torch.float32, device=device)
        d["dW_r"] = torch.empty(E, H, dtype=torch.float32, device=device)
        d["router_ws"] = torch.empty(max(lib.moe_router_workspace_bytes(T, H, E), 1), dtype=torch.uint8,
                                     device=device)
    return d
