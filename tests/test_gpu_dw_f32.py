"""fp32 weight gradients (moe_layer_bwd_dw_f32 / moe_layer_bwd_x_dw_f32).

The wgrad GEMMs store their fp32 accumulators unrounded. Pinned three ways:
against the oracle within the float tolerance; against the bf16 entry point
(the same accumulators rounded once to bf16, so bit-equal); and accumulate
mode equal to the fp32 sum dW0 + dW done by torch (one IEEE add per element,
so bit-equal). Experts without rows: zeros, or unchanged when accumulating.
"""
import pytest
import torch

from routed_grouped_gemm_router_b200 import layer
from routed_grouped_gemm_router_b200.inputs import WORKLOADS, make_inputs, small_inputs

import gpu_util as U

pytestmark = pytest.mark.gpu


def _bufs(st, grads_dtype, H, I, dW0=None):
    E = st.E
    dev = st.Y.device
    g = dict(dX=torch.empty(st.T, H, dtype=torch.bfloat16, device=dev),
             dlogits=torch.empty(st.T, E, dtype=torch.float32, device=dev))
    if dW0 is not None:
        g["dW_gu"], g["dW_d"] = dW0[0].clone(), dW0[1].clone()
    else:
        g["dW_gu"] = torch.full((E, 2 * I, H), float("nan"), dtype=grads_dtype, device=dev)
        g["dW_d"] = torch.full((E, H, I), float("nan"), dtype=grads_dtype, device=dev)
    return {"grads": g}


def _three_ways(inp, k, gather):
    """bf16 grads, fp32 grads, and fp32 grads accumulated onto dW0."""
    d = U.to_dev(inp)
    H, I = inp.W_gu.shape[2], inp.W_d.shape[2]
    st = layer.forward(d["logits"], d["X"], d["W_gu"], d["W_d"], k, gather=gather)
    g16 = layer.backward(st, d["dY"], d["W_gu"], d["W_d"], bufs=_bufs(st, torch.bfloat16, H, I))
    g32 = layer.backward(st, d["dY"], d["W_gu"], d["W_d"], bufs=_bufs(st, torch.float32, H, I))
    gen = torch.Generator(device="cuda").manual_seed(5)
    dW0 = (torch.randn(st.E, 2 * I, H, generator=gen, device="cuda") * 1e-2,
           torch.randn(st.E, H, I, generator=gen, device="cuda") * 1e-2)
    gacc = layer.backward(st, d["dY"], d["W_gu"], d["W_d"], bufs=_bufs(st, torch.float32, H, I, dW0),
                          accumulate=True)
    assert U.B.last_device_status() == 0
    return st, g16, g32, gacc, dW0


@pytest.mark.parametrize("gather", [False, True], ids=["permuted", "gathered"])
@pytest.mark.parametrize("shape", [(600, 256, 16, 4, 192, 0), (333, 200, 12, 3, 72, 3), (97, 64, 8, 2, 24, 5)],
                         ids=lambda s: "T%d_H%d_E%d_k%d_I%d_dead%d" % s)
def test_dw_f32_matches_oracle_and_bf16(shape, gather):
    T, H, E, k, I, dead = shape
    # dead experts are made by the stress bias, which comes with a Zipf skew
    inp = small_inputs(T, H, E, k, I, seed=T + H, zipf_s=1.0 if dead else 0.0, dead=dead)
    st, g16, g32, gacc, dW0 = _three_ways(inp, k, gather)
    _, bwd = U.oracle_full(inp, k)
    for name in ("dW_gu", "dW_d"):
        assert g32[name].dtype == torch.float32
        U.assert_rel(U.to_np(g32[name]), bwd[name], name + " (fp32)")
        assert torch.equal(g32[name].bfloat16(), g16[name]), name + ": bf16(fp32 output) != bf16 output"
    assert torch.equal(gacc["dW_gu"], dW0[0] + g32["dW_gu"])
    assert torch.equal(gacc["dW_d"], dW0[1] + g32["dW_d"])
    # the rest of the backward does not depend on the weight-gradient format
    for name in ("dX", "dlogits"):
        assert torch.equal(g32[name], g16[name]) and torch.equal(gacc[name], g16[name]), name
    counts = U.to_np(st.perm["counts"])
    empty = [e for e in range(E) if counts[e] == 0]
    assert len(empty) >= dead
    for e in empty:
        assert (g32["dW_gu"][e] == 0).all() and (g32["dW_d"][e] == 0).all()
        assert torch.equal(gacc["dW_gu"][e], dW0[0][e]) and torch.equal(gacc["dW_d"][e], dW0[1][e])


def test_dw_f32_empty_batch():
    E, H, I, k = 8, 64, 32, 2
    logits = torch.empty(0, E, device="cuda")
    X = torch.empty(0, H, dtype=torch.bfloat16, device="cuda")
    dY = torch.empty(0, H, dtype=torch.bfloat16, device="cuda")
    W_gu = torch.randn(E, 2 * I, H, device="cuda").bfloat16()
    W_d = torch.randn(E, H, I, device="cuda").bfloat16()
    st = layer.forward(logits, X, W_gu, W_d, k)
    g = layer.backward(st, dY, W_gu, W_d, bufs=_bufs(st, torch.float32, H, I))
    assert (g["dW_gu"] == 0).all() and (g["dW_d"] == 0).all()
    dW0 = (torch.ones(E, 2 * I, H, device="cuda"), torch.ones(E, H, I, device="cuda"))
    g = layer.backward(st, dY, W_gu, W_d, bufs=_bufs(st, torch.float32, H, I, dW0), accumulate=True)
    assert (g["dW_gu"] == 1).all() and (g["dW_d"] == 1).all()
    assert U.B.last_device_status() == 0


def test_dw_f32_full_size_rounds_to_bf16_output():
    """Full-size Qwen3-30B-A3B-shaped layer: fp32 weight gradients rounded to
    bf16 equal the bf16 entry point's bit for bit (a property that holds at
    any size), and accumulating twice from zero gives exactly 2 x dW."""
    wl = WORKLOADS["qwen3-30b-a3b"]
    inp = make_inputs(wl, seed=0)
    d = U.to_dev(inp)
    st = layer.forward(d["logits"], d["X"], d["W_gu"], d["W_d"], wl.k)
    g16 = layer.backward(st, d["dY"], d["W_gu"], d["W_d"], bufs=_bufs(st, torch.bfloat16, wl.H, wl.I))
    zeros = (torch.zeros(wl.E, 2 * wl.I, wl.H, device="cuda"), torch.zeros(wl.E, wl.H, wl.I, device="cuda"))
    b = _bufs(st, torch.float32, wl.H, wl.I, zeros)
    g32 = layer.backward(st, d["dY"], d["W_gu"], d["W_d"], bufs=b, accumulate=True)
    for name in ("dW_gu", "dW_d"):
        assert torch.equal(g32[name].bfloat16(), g16[name]), name
    once = (g32["dW_gu"].clone(), g32["dW_d"].clone())
    layer.backward(st, d["dY"], d["W_gu"], d["W_d"], bufs=b, accumulate=True)
    assert torch.equal(b["grads"]["dW_gu"], 2 * once[0]) and torch.equal(b["grads"]["dW_d"], 2 * once[1])
    assert U.B.last_device_status() == 0
