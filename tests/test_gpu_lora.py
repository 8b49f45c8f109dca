"""LoRA adapters on the stacked expert weights, on the GPU through the C ABI
(moe_experts_fwd_lora / moe_layer_bwd_lora) against the oracle (the layer on
W + scale B A, adapter gradients by the chain rule). Also: B = 0 gives the
base layer bit for bit, accumulate mode adds exactly, the base weights'
gradients when asked for, the empty batch, and a full-size layer."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as orc
from routed_grouped_gemm_router_b200 import binding as B
from routed_grouped_gemm_router_b200 import layer
from routed_grouped_gemm_router_b200.inputs import WORKLOADS, make_inputs, make_lora, small_inputs

import gpu_util as U

pytestmark = pytest.mark.gpu

SCALE = 2.0


def _dev_lora(ad, scale=SCALE):
    d = {n: t.cuda() for n, t in ad.items()}
    d["scale"] = scale
    return d


def _run(inp, k, lora, accumulate_onto=None, base_grads=False, save_gu=True):
    d = U.to_dev(inp)
    st = layer.forward_lora(d["logits"], d["X"], d["W_gu"], d["W_d"], k, lora, save_gu=save_gu)
    bufs = None
    if accumulate_onto is not None:
        bufs = {"grads": {n: t.clone() for n, t in accumulate_onto.items()}}
    g = layer.backward_lora(st, d["dY"], d["W_gu"], d["W_d"], bufs=bufs, accumulate=accumulate_onto is not None,
                            base_grads=base_grads)
    assert B.last_device_status() == 0
    return st, g


CASES = [(600, 256, 16, 4, 192, 16, 0), (333, 200, 12, 3, 72, 8, 3), (257, 128, 8, 2, 96, 64, 0),
         (130, 64, 5, 2, 40, 72, 0), (700, 320, 13, 3, 136, 24, 2), (1, 64, 4, 2, 32, 8, 0),
         # the largest rank (8 extension K blocks; 256-wide tiles, two N tiles in every skinny product)
         (300, 128, 40, 4, 64, 512, 0),
         # sizes that are not multiples of 64 (as in gpt-oss, H = I = 2880), rank 128
         (420, 288, 9, 3, 288, 128, 0)]


@pytest.mark.parametrize("shape", CASES, ids=lambda s: "T%d_H%d_E%d_k%d_I%d_r%d_dead%d" % s)
def test_lora_matches_oracle(shape):
    T, H, E, k, I, r, dead = shape
    inp = small_inputs(T, H, E, k, I, seed=T + r, zipf_s=1.0 if dead else 0.0, dead=dead)
    ad = make_lora(E, H, I, r, seed=r)
    st, g = _run(inp, k, _dev_lora(ad), base_grads=True)
    a = {n: t.double().numpy() for n, t in ad.items()}
    fwd = orc.lora_layer_forward(inp.logits, inp.X, inp.W_gu, inp.W_d, k, a["A_gu"], a["B_gu"], a["A_d"], a["B_d"],
                                 SCALE)
    bwd = orc.lora_layer_backward(fwd, inp.dY, inp.X, k, a["A_gu"], a["B_gu"], a["A_d"], a["B_d"], SCALE)
    U.check_routing_exact(st, fwd)
    U.assert_rel(U.to_np(st.Y), fwd["Y"], "Y")
    U.assert_rel(U.to_np(st.Z_gu), SCALE * np.concatenate(
        [inp.X.double().numpy()[fwd["sorted_pair"][fwd["offsets"][e]:fwd["offsets"][e + 1]] // k] @ a["A_gu"][e].T
         for e in range(E)], axis=0).reshape(-1, r), "Z_gu")
    for name in ("dX", "dlogits", "dA_gu", "dB_gu", "dA_d", "dB_d", "dW_gu", "dW_d"):
        U.assert_rel(U.to_np(g[name]), bwd[name], name)
    counts = fwd["counts"]
    for e in np.nonzero(counts == 0)[0]:
        for name in ("dA_gu", "dB_gu", "dA_d", "dB_d", "dW_gu", "dW_d"):
            assert (U.to_np(g[name][int(e)]) == 0).all(), (name, e)


def test_lora_zero_B_is_the_base_layer_bit_for_bit():
    """B = 0: each GEMM's extra K blocks add exact zeros to its accumulator,
    so Y, dX, dlogits and the base weight gradients equal the plain layer's
    bit for bit, and dA = 0 exactly."""
    T, H, E, k, I, r = 500, 256, 12, 4, 160, 16
    inp = small_inputs(T, H, E, k, I, seed=9)
    ad = make_lora(E, H, I, r, seed=1)
    ad["B_gu"].zero_()
    ad["B_d"].zero_()
    st, g = _run(inp, k, _dev_lora(ad), base_grads=True)
    st0, g0 = U.run_layer(inp, k)
    assert torch.equal(st.Y, st0.Y) and torch.equal(st.h, st0.h) and torch.equal(st.O, st0.O)
    for name in ("dX", "dlogits", "dW_gu", "dW_d"):
        assert torch.equal(g[name], g0[name]), name
    assert (g["dA_gu"] == 0).all() and (g["dA_d"] == 0).all()
    assert g["dB_gu"].abs().max() > 0 and g["dB_d"].abs().max() > 0


def test_lora_accumulate_recompute_and_determinism():
    T, H, E, k, I, r = 400, 192, 10, 3, 104, 32
    inp = small_inputs(T, H, E, k, I, seed=4, zipf_s=1.0, dead=2)
    lora = _dev_lora(make_lora(E, H, I, r, seed=2))
    st, g = _run(inp, k, lora)
    _, g2 = _run(inp, k, lora)
    for n in g:
        assert torch.equal(g[n], g2[n]), n  # deterministic: no atomics anywhere
    gen = torch.Generator(device="cuda").manual_seed(3)
    base = {n: torch.randn(g[n].shape, generator=gen, device="cuda") for n in ("dA_gu", "dB_gu", "dA_d", "dB_d")}
    _, ga = _run(inp, k, lora, accumulate_onto=base)
    for n in base:
        assert torch.equal(ga[n], base[n] + g[n]), n
    # g|u recomputed in the backward instead of saved: the same results
    _, gr = _run(inp, k, lora, save_gu=False)
    for n in g:
        assert torch.equal(gr[n], g[n]), n


def test_lora_empty_batch():
    E, H, I, k, r = 8, 64, 32, 2, 16
    lora = _dev_lora(make_lora(E, H, I, r, seed=0))
    logits = torch.empty(0, E, device="cuda")
    X = torch.empty(0, H, dtype=torch.bfloat16, device="cuda")
    W_gu = torch.randn(E, 2 * I, H, device="cuda").bfloat16()
    W_d = torch.randn(E, H, I, device="cuda").bfloat16()
    st = layer.forward_lora(logits, X, W_gu, W_d, k, lora)
    g = layer.backward_lora(st, torch.empty(0, H, dtype=torch.bfloat16, device="cuda"), W_gu, W_d)
    for n in ("dA_gu", "dB_gu", "dA_d", "dB_d"):
        assert (g[n] == 0).all(), n
    ones = {n: torch.ones_like(g[n]) for n in ("dA_gu", "dB_gu", "dA_d", "dB_d")}
    g = layer.backward_lora(st, torch.empty(0, H, dtype=torch.bfloat16, device="cuda"), W_gu, W_d,
                            bufs={"grads": ones}, accumulate=True)
    for n in ones:
        assert (g[n] == 1).all(), n
    assert B.last_device_status() == 0


class _EffWeights:
    """W[e] + scale B[e] A[e] for one expert at a time (oracle arithmetic on
    one expert's slices), indexable like the stacked weights."""

    def __init__(self, W, A, Bm, which):
        self.W, self.A, self.B, self.which = W, A, Bm, which

    def __getitem__(self, e):
        e = int(e)
        one = lambda t: t[e:e + 1].double().numpy()
        if self.which == "gu":
            w, _ = orc.lora_effective_weights(one(self.W), np.zeros((1, 8, 1)), one(self.A), one(self.B),
                                              np.zeros((1, 1, 1)), np.zeros((1, 8, 1)), SCALE)
        else:
            _, w = orc.lora_effective_weights(np.zeros((1, 8, 1)), one(self.W), np.zeros((1, 1, 1)),
                                              np.zeros((1, 8, 1)), one(self.A), one(self.B), SCALE)
        return w[0]


def test_lora_full_size():
    """Qwen3-30B-A3B-shaped layer with rank-16 adapters: routing bit-exact,
    sampled tokens' Y / dX / dlogits and sampled experts' adapter gradients
    against the oracle one token / one expert at a time."""
    wl = WORKLOADS["qwen3-30b-a3b"]
    k, r = wl.k, 16
    inp = make_inputs(wl, seed=0, with_dy=True)
    ad = make_lora(wl.E, wl.H, wl.I, r, seed=5)
    st, g = _run(inp, k, _dev_lora(ad))
    idx, w, probs = orc.route(inp.logits, k)
    counts, offsets, sorted_pair, pair_pos = orc.permute(idx, wl.E)
    U.check_routing_exact(st, dict(idx=idx, w=w, probs=probs, counts=counts, offsets=offsets,
                                   sorted_pair=sorted_pair, pair_pos=pair_pos))
    Wgu = _EffWeights(inp.W_gu, ad["A_gu"], ad["B_gu"], "gu")
    Wd = _EffWeights(inp.W_d, ad["A_d"], ad["B_d"], "d")
    rng = np.random.default_rng(1)
    toks = sorted(set(rng.choice(wl.T, 24, replace=False).tolist() + [0, wl.T - 1]))
    U.assert_rel(U.to_np(st.Y[toks]), orc.token_forward(toks, idx, w, inp.X, Wgu, Wd), "Y")
    tb = orc.token_backward(toks, idx, w, probs, inp.dY, inp.X, Wgu, Wd)
    U.assert_rel(U.to_np(g["dX"][toks]), tb["dX"], "dX")
    U.assert_rel(U.to_np(g["dlogits"][toks]), tb["dlogits"], "dlogits")
    live = np.nonzero(counts)[0]
    for e in sorted({int(live[0]), int(np.argmax(counts)), int(live[-1])}):
        G_gu, G_d = orc.expert_weight_grads(e, offsets, sorted_pair, w, inp.dY, inp.X, Wgu, Wd, k)
        Bgu, Agu = ad["B_gu"][e].double().numpy(), ad["A_gu"][e].double().numpy()
        Bd, Ad = ad["B_d"][e].double().numpy(), ad["A_d"][e].double().numpy()
        U.assert_rel(U.to_np(g["dA_gu"][e]), SCALE * Bgu.T @ G_gu, f"dA_gu[{e}]")
        U.assert_rel(U.to_np(g["dB_gu"][e]), SCALE * G_gu @ Agu.T, f"dB_gu[{e}]")
        U.assert_rel(U.to_np(g["dA_d"][e]), SCALE * Bd.T @ G_d, f"dA_d[{e}]")
        U.assert_rel(U.to_np(g["dB_d"][e]), SCALE * G_d @ Ad.T, f"dB_d[{e}]")
