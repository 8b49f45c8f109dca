"""Seeded synthetic inputs for the MoE expert layer.

This module only draws random numbers and rounds them to the storage dtypes; it
holds none of the layer's arithmetic. Both the CUDA path (through the binding)
and the CPU oracle are fed from here, so the two always see identical inputs.

Shapes and distributions follow the layers the pages discuss:
  * Qwen3-MoE (30B-A3B, 235B-A22B) and GPT-OSS-20b expert layers
    (axolotl issue #3155, "Feature description"; torchtune PR #2820, opening
    comment; unsloth PR #3812, stacked weight shapes ``[E, 2I, H]`` and
    ``[E, H, I]``).
  * activations ~ N(0, 1) stored as bf16, expert weights ~ N(0, 0.02) stored as
    bf16, router weight ~ N(0, 0.02) in fp32, upstream gradient ~ N(0, 1) bf16.
  * router logits come from the caller-side fp32 ``Linear(H -> E)``
    (weight ``[E, H]``, axolotl issue #3155, router-shape discussion),
    computed here once on the CPU so both sides receive the same fp32 tensor.

Draw order from one ``torch.Generator`` seeded with ``seed``:
X, W_r, W_gate, W_up, W_down, dY, then (stress workloads only) the expert
permutation of the popularity bias.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    """One expert-layer problem size. P = T * k routed (token, expert) pairs."""

    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    zipf_s: float = 0.0      # > 0: add the Zipf popularity bias to the logits
    dead_experts: int = 0    # experts forced to receive no tokens (stress bias)
    backward: bool = True

    @property
    def P(self) -> int:
        return self.T * self.k

    def flops_fwd(self) -> float:
        """Useful forward flops: gate/up (4·H·I) + down (2·H·I) per pair."""
        return 6.0 * self.H * self.I * self.P

    def flops_bwd(self) -> float:
        """Useful backward flops: dgrad (6·H·I) + wgrad (6·H·I) per pair."""
        return 12.0 * self.H * self.I * self.P


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", T=256, H=128, E=8, k=2, I=256),
        Workload("qwen3-30b-a3b", T=8192, H=2048, E=128, k=8, I=768),
        Workload("gpt-oss-20b", T=16384, H=2880, E=32, k=4, I=2880),
        Workload("qwen3-235b-a22b", T=16384, H=4096, E=128, k=8, I=1536),
        Workload("zipf-t64", T=64, H=2048, E=128, k=8, I=768, zipf_s=1.2, dead_experts=20),
        Workload("zipf-t32768", T=32768, H=2048, E=128, k=8, I=768, zipf_s=1.2, dead_experts=20),
    ]
}


@dataclass
class LayerInputs:
    """Host (CPU) tensors of one problem. bf16 tensors are already rounded."""

    wl: Workload
    X: torch.Tensor          # [T, H] bf16
    W_r: torch.Tensor        # [E, H] fp32 (caller-side router weight)
    W_gu: torch.Tensor       # [E, 2I, H] bf16, rows [0, I) gate, [I, 2I) up
    W_d: torch.Tensor        # [E, H, I] bf16
    logits: torch.Tensor     # [T, E] fp32
    dY: torch.Tensor | None  # [T, H] bf16
    bias: torch.Tensor | None = field(default=None)  # [E] fp32 stress bias


def zipf_bias(E: int, s: float, dead: int, gen: torch.Generator) -> torch.Tensor:
    """Per-expert additive logit bias: a seeded random ranking of the experts,
    ``dead`` of them pushed to -1e4 (they then receive no tokens while at least
    k experts stay live), the rest given ln of a Zipf(s) probability by rank."""
    perm = torch.randperm(E, generator=gen)
    live = E - dead
    harmonic = sum(r ** (-s) for r in range(1, live + 1))
    bias = torch.empty(E, dtype=torch.float32)
    for rank, e in enumerate(perm.tolist()):
        if rank < live:
            bias[e] = math.log((rank + 1) ** (-s) / harmonic)
        else:
            bias[e] = -1.0e4
    return bias


def make_inputs(wl: Workload, seed: int = 0, with_dy: bool | None = None) -> LayerInputs:
    """Draw one problem on the CPU (bf16-rounded) from ``seed``."""
    if with_dy is None:
        with_dy = wl.backward
    g = torch.Generator().manual_seed(seed)
    T, H, E, I = wl.T, wl.H, wl.E, wl.I
    X = torch.randn(T, H, generator=g).to(torch.bfloat16)
    W_r = torch.randn(E, H, generator=g) * 0.02
    W_gate = (torch.randn(E, I, H, generator=g) * 0.02).to(torch.bfloat16)
    W_up = (torch.randn(E, I, H, generator=g) * 0.02).to(torch.bfloat16)
    W_d = (torch.randn(E, H, I, generator=g) * 0.02).to(torch.bfloat16)
    dY = torch.randn(T, H, generator=g).to(torch.bfloat16) if with_dy else None
    W_gu = torch.cat([W_gate, W_up], dim=1).contiguous()
    del W_gate, W_up
    bias = zipf_bias(E, wl.zipf_s, wl.dead_experts, g) if wl.zipf_s > 0 else None
    logits = router_logits(X, W_r, bias)
    return LayerInputs(wl, X, W_r, W_gu, W_d, logits, dY, bias)


def router_logits(X: torch.Tensor, W_r: torch.Tensor, bias: torch.Tensor | None) -> torch.Tensor:
    """Caller-side router Linear in fp32 on the CPU (not part of the layer)."""
    logits = X.float() @ W_r.t()
    if bias is not None:
        logits = logits + bias
    return logits.contiguous()


def make_lora(E: int, H: int, I: int, r: int, seed: int = 0, std: float = 0.02) -> dict:
    """Seeded LoRA adapters for the stacked expert weights, bf16-rounded:
    A_gu [E, r, H], B_gu [E, 2I, r], A_d [E, r, I], B_d [E, H, r], entries
    N(0, std) (B nonzero, unlike a fresh adapter, so that the term is
    exercised)."""
    g = torch.Generator().manual_seed(seed)
    return dict(A_gu=(torch.randn(E, r, H, generator=g) * std).to(torch.bfloat16),
                B_gu=(torch.randn(E, 2 * I, r, generator=g) * std).to(torch.bfloat16),
                A_d=(torch.randn(E, r, I, generator=g) * std).to(torch.bfloat16),
                B_d=(torch.randn(E, H, r, generator=g) * std).to(torch.bfloat16))


def small_inputs(T, H, E, k, I, seed=0, with_dy=True, zipf_s=0.0, dead=0) -> LayerInputs:
    """Convenience: an ad-hoc problem size (test shapes)."""
    return make_inputs(Workload("adhoc", T, H, E, k, I, zipf_s=zipf_s, dead_experts=dead),
                       seed=seed, with_dy=with_dy)
