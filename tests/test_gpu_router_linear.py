"""Router Linear on the GPU (moe_router_fwd / moe_router_bwd through the C
ABI) against the oracle: logits = X W_r^T to fp32 accuracy, routing
bit-exact given the GPU's logits (and equal to the oracle's own routing
wherever the float64 logits are not within rounding of a tie), dW_r and the
router's share of dX; the whole block fwd+bwd with the router inside."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as orc
from routed_grouped_gemm_router_b200 import binding as B
from routed_grouped_gemm_router_b200 import layer
from routed_grouped_gemm_router_b200.inputs import WORKLOADS, make_inputs, small_inputs

import gpu_util as U

pytestmark = pytest.mark.gpu

# fp32-class accuracy of the logits and dW_r: exact products summed in fp32.
# A bf16-only product would miss by ~1e-3 of max|ref|.
LOGIT_TOL = 2e-5
DWR_TOL = 1e-4


def router_inputs(T, H, E, seed):
    g = torch.Generator().manual_seed(seed)
    X = torch.randn(T, H, generator=g).bfloat16()
    W_r = torch.randn(E, H, generator=g) * 0.02
    dl = torch.randn(T, E, generator=g) * 1e-2
    dX0 = torch.randn(T, H, generator=g).bfloat16()
    return X, W_r, dl, dX0


def check_forward(X, W_r, k, out):
    logits = U.to_np(out["logits"]).astype(np.float64)
    ref = orc.router_logits(X.float().numpy(), W_r.numpy())
    U.assert_rel(logits, ref, "logits", tol=LOGIT_TOL)
    # routing: bit-exact given the GPU's fp32 logits
    gl = out["logits"].cpu().numpy()
    idx, w, probs = orc.route(gl, k)
    assert (U.to_np(out["topk_idx"]) == idx).all()
    np.testing.assert_allclose(U.to_np(out["topk_w"]), w, atol=U.W_ABS_TOL, rtol=0)
    np.testing.assert_allclose(U.to_np(out["probs"]), probs, atol=1e-6, rtol=1e-4)
    # and the oracle's own routing on its float64 logits wherever no two of a
    # token's k+1 leading logits are within the logits' error bound
    ridx = orc.select_topk(ref, k)
    E = ref.shape[1]
    srt = -np.sort(-ref, axis=1)[:, :min(k + 1, E)]
    gap = np.abs(np.diff(srt, axis=1)).min(axis=1) if srt.shape[1] > 1 else np.full(len(ref), np.inf)
    clear = gap > 4 * LOGIT_TOL * np.abs(ref).max()
    assert clear.mean() > 0.9
    assert (U.to_np(out["topk_idx"])[clear] == ridx[clear]).all()


@pytest.mark.parametrize("shape", [(256, 128, 8, 2), (300, 200, 6, 2), (700, 320, 13, 3), (1, 64, 4, 2),
                                   (3, 72, 5, 2), (1200, 512, 33, 4), (96, 128, 1000, 8), (64, 256, 1024, 8),
                                   (500, 8, 3, 1), (130, 2048, 1, 1), (2048, 2048, 128, 8)],
                         ids=lambda s: "T%d_H%d_E%d_k%d" % s)
def test_router_fwd_bwd_matches_oracle(shape):
    T, H, E, k = shape
    X, W_r, dl, dX0 = router_inputs(T, H, E, seed=sum(shape))
    out = B.moe_router_fwd(X.cuda(), W_r.cuda(), k)
    dX = dX0.cuda().clone()
    dW_r, dX = B.moe_router_bwd(dl.cuda(), X.cuda(), W_r.cuda(), dX=dX)
    assert B.last_device_status() == 0
    check_forward(X, W_r, k, out)
    rdW, rdX = orc.router_logits_backward(dl.numpy(), X.float().numpy(), W_r.numpy())
    U.assert_rel(U.to_np(dW_r), rdW, "dW_r", tol=DWR_TOL)
    ref = dX0.double().numpy() + rdX
    err = np.abs(U.to_np(dX) - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2e-4 * np.abs(ref).max()
    assert (err <= bound).all(), f"dX: worst excess {(err - bound).max():.3e}"


def test_router_bwd_outputs_are_optional_and_deterministic():
    T, H, E = 777, 384, 40
    X, W_r, dl, dX0 = router_inputs(T, H, E, seed=4)
    Xc, Wc, dlc = X.cuda(), W_r.cuda(), dl.cuda()
    dW_a, _ = B.moe_router_bwd(dlc, Xc, Wc)
    dW_b, _ = B.moe_router_bwd(dlc, Xc, Wc)
    assert torch.equal(dW_a, dW_b)
    dX = dX0.cuda().clone()
    none, dX = B.moe_router_bwd(dlc, Xc, Wc, dX=dX, want_dW_r=False)
    assert none is None
    dX2 = dX0.cuda().clone()
    B.moe_router_bwd(dlc, Xc, Wc, dX=dX2, want_dW_r=False)
    assert torch.equal(dX, dX2)
    a = B.moe_router_fwd(Xc, Wc, 4)
    b = B.moe_router_fwd(Xc, Wc, 4)
    assert torch.equal(a["logits"], b["logits"]) and torch.equal(a["topk_idx"], b["topk_idx"])
    assert B.last_device_status() == 0


def test_router_empty_batch():
    E, H = 8, 64
    X = torch.empty(0, H, dtype=torch.bfloat16, device="cuda")
    W_r = torch.randn(E, H, device="cuda")
    out = B.moe_router_fwd(X, W_r, 2)
    assert out["topk_idx"].shape == (0, 2)
    dW = torch.full((E, H), 7.0, device="cuda")
    B.moe_router_bwd(torch.empty(0, E, device="cuda"), X, W_r, dW_r=dW)
    assert (dW == 0).all() and B.last_device_status() == 0


def test_block_with_router_matches_oracle():
    """X, W_r -> router -> experts -> combine; backward with the router's dX
    share added in place and dW_r; routing compared bit-exactly given the
    GPU's logits, gradients against the oracle on those logits."""
    T, H, E, k, I = 600, 256, 16, 4, 192
    inp = small_inputs(T, H, E, k, I, seed=12)
    d = U.to_dev(inp)
    W_r = inp.W_r.cuda()
    r = B.moe_router_fwd(d["X"], W_r, k)
    st = layer.forward(r["logits"], d["X"], d["W_gu"], d["W_d"], k)
    grads = layer.backward(st, d["dY"], d["W_gu"], d["W_d"])
    dW_r, dX = B.moe_router_bwd(grads["dlogits"], d["X"], W_r, dX=grads["dX"])
    assert B.last_device_status() == 0
    gl = r["logits"].cpu().numpy()
    U.assert_rel(gl, orc.router_logits(inp.X, inp.W_r), "logits", tol=LOGIT_TOL)
    fwd = orc.layer_forward(gl, inp.X, inp.W_gu, inp.W_d, k)
    bwd = orc.layer_backward(fwd, inp.dY, inp.X, inp.W_gu, inp.W_d, k)
    rdW, rdX = orc.router_logits_backward(bwd["dlogits"], inp.X, inp.W_r)
    U.check_routing_exact(st, fwd)
    U.assert_rel(U.to_np(st.Y), fwd["Y"], "Y")
    U.assert_rel(U.to_np(dX), bwd["dX"] + rdX, "dX (experts + router)")
    U.assert_rel(U.to_np(dW_r), rdW, "dW_r")


@pytest.mark.parametrize("name", ["qwen3-30b-a3b", "gpt-oss-20b"])
def test_router_full_size(name):
    """Full-size router on the bench's layer shapes: every logit, dW_r and dX
    element against the oracle (these products are cheap in float64)."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl, seed=0)
    g = torch.Generator().manual_seed(99)
    dl = torch.randn(wl.T, wl.E, generator=g) * 1e-2
    Xc, Wc = inp.X.cuda(), inp.W_r.cuda()
    out = B.moe_router_fwd(Xc, Wc, wl.k)
    dX = inp.dY.cuda().clone()  # any bf16 [T, H] serves as the incoming dX
    dW_r, dX = B.moe_router_bwd(dl.cuda(), Xc, Wc, dX=dX)
    assert B.last_device_status() == 0
    check_forward(inp.X, inp.W_r, wl.k, out)
    rdW, rdX = orc.router_logits_backward(dl.numpy(), inp.X.float().numpy(), inp.W_r.numpy())
    U.assert_rel(U.to_np(dW_r), rdW, "dW_r", tol=DWR_TOL)
    ref = inp.dY.double().numpy() + rdX
    err = np.abs(U.to_np(dX) - ref)
    assert (err <= 2.0 ** -8 * np.abs(ref) + 2e-4 * np.abs(ref).max()).all()
