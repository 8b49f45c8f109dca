"""Pins of the oracle's forward against a dense brute-force evaluation, closed
forms and special cases that reduce to a single SwiGLU MLP. CPU only."""
import math

import numpy as np
import pytest
import torch

from oracle import moe_oracle as orc
from routed_grouped_gemm_router_b200.inputs import small_inputs


def _silu(x):
    return x / (1.0 + math.exp(-x))


def dense_bruteforce(logits, X, W_gu, W_d, k):
    """Every token through every expert in scalar Python loops, weighted by a
    dense [T, E] matrix that holds the renormalised top-k softmax weight of the
    selected experts and zero elsewhere. Selection by counting how many experts
    beat each one (larger logit, or equal logit and smaller index)."""
    l = np.asarray(logits, dtype=np.float32)
    X = np.asarray(X, dtype=np.float64)
    W_gu = np.asarray(W_gu, dtype=np.float64)
    W_d = np.asarray(W_d, dtype=np.float64)
    T, H = X.shape
    E, twoI, _ = W_gu.shape
    I = twoI // 2
    Y = np.zeros((T, H))
    for t in range(T):
        z = [math.exp(float(l[t, e]) - float(l[t].max())) for e in range(E)]
        p = [ze / sum(z) for ze in z]
        sel = [e for e in range(E)
               if sum(1 for f in range(E) if l[t, f] > l[t, e] or (l[t, f] == l[t, e] and f < e)) < k]
        S = sum(p[e] for e in sel) + 1e-20
        for e in range(E):
            wte = p[e] / S if e in sel else 0.0
            hvec = []
            for i in range(I):
                g = sum(X[t, c] * W_gu[e, i, c] for c in range(H))
                u = sum(X[t, c] * W_gu[e, I + i, c] for c in range(H))
                hvec.append(_silu(g) * u)
            for c in range(H):
                Y[t, c] += wte * sum(hvec[i] * W_d[e, c, i] for i in range(I))
    return Y


@pytest.mark.parametrize("T,H,E,k,I,seed", [(5, 4, 3, 2, 3, 0), (6, 3, 4, 1, 2, 1), (4, 5, 4, 4, 2, 2)])
def test_forward_matches_dense_bruteforce(T, H, E, k, I, seed):
    inp = small_inputs(T, H, E, k, I, seed=seed)
    W_gu = inp.W_gu.float().numpy() * 20  # larger weights so silu is far from linear
    W_d = inp.W_d.float().numpy() * 20
    fwd = orc.layer_forward(inp.logits, inp.X, W_gu, W_d, k)
    ref = dense_bruteforce(inp.logits.numpy(), inp.X.float().numpy(), W_gu, W_d, k)
    np.testing.assert_allclose(fwd["Y"], ref, rtol=1e-10, atol=1e-12)


def test_scalar_layer_closed_form():
    """T=1, H=I=1, two experts, k=2, logits (0, ln 3) -> p = (1/4, 3/4).
    Expert 0: g = 2*0.5 = 1, u = 2*1.5 = 3, o = 2*silu(1)*3.
    Expert 1: g = 2*(-1) = -2, u = 2*0.25 = 0.5, o = 4*silu(-2)*0.5.
    Y = 3/4 * o_1 + 1/4 * o_0 = -3/(1+e^2) + 1.5/(1+e^-1)."""
    logits = np.array([[0.0, math.log(3.0)]], dtype=np.float32)
    X = np.array([[2.0]])
    W_gu = np.array([[[0.5], [1.5]], [[-1.0], [0.25]]])   # [E=2, 2I=2, H=1]
    W_d = np.array([[[2.0]], [[4.0]]])                    # [E=2, H=1, I=1]
    fwd = orc.layer_forward(logits, X, W_gu, W_d, 2)
    y_ref = -3.0 / (1.0 + math.exp(2.0)) + 1.5 / (1.0 + math.exp(-1.0))
    p1 = float(np.exp(np.float64(np.float32(math.log(3.0)))))  # fp32-rounded ln 3
    w1 = p1 / (1 + p1)
    y_ref_exact_w = w1 * (-4.0 / (1.0 + math.exp(2.0))) + (1 - w1) * (6.0 / (1.0 + math.exp(-1.0)))
    assert fwd["idx"].tolist() == [[1, 0]]
    assert abs(fwd["Y"][0, 0] - y_ref_exact_w) < 1e-14
    assert abs(fwd["Y"][0, 0] - y_ref) < 1e-6


def _swiglu_mlp_torch(X, W_gu_e, W_d_e):
    X = torch.as_tensor(X, dtype=torch.float64)
    Wg, Wu = torch.as_tensor(W_gu_e, dtype=torch.float64).chunk(2, dim=0)
    Wd = torch.as_tensor(W_d_e, dtype=torch.float64)
    return (torch.nn.functional.silu(X @ Wg.T) * (X @ Wu.T)) @ Wd.T


def test_identical_experts_reduce_to_one_mlp():
    inp = small_inputs(32, 16, 6, 3, 24, seed=7)
    W_gu = inp.W_gu.float().numpy()
    W_d = inp.W_d.float().numpy()
    W_gu[:] = W_gu[0]
    W_d[:] = W_d[0]
    fwd = orc.layer_forward(inp.logits, inp.X, W_gu, W_d, 3)
    ref = _swiglu_mlp_torch(inp.X.float().numpy(), W_gu[0], W_d[0]).numpy()
    np.testing.assert_allclose(fwd["Y"], ref, rtol=1e-10, atol=1e-13)


def test_one_hot_logits_pick_single_expert():
    inp = small_inputs(12, 8, 4, 1, 8, seed=8)
    logits = np.full((12, 4), -5.0, dtype=np.float32)
    choice = np.arange(12) % 4
    logits[np.arange(12), choice] = 5.0
    W_gu = inp.W_gu.float().numpy()
    W_d = inp.W_d.float().numpy()
    fwd = orc.layer_forward(logits, inp.X, W_gu, W_d, 1)
    X = inp.X.float().numpy()
    for t in range(12):
        ref = _swiglu_mlp_torch(X[t:t + 1], W_gu[choice[t]], W_d[choice[t]]).numpy()[0]
        np.testing.assert_allclose(fwd["Y"][t], ref, rtol=1e-10, atol=1e-13)


def test_E_equals_k_weights_are_softmax_and_zero_down_gives_zero():
    inp = small_inputs(10, 8, 4, 4, 8, seed=9)
    fwd = orc.layer_forward(inp.logits, inp.X, inp.W_gu, inp.W_d, 4)
    p = torch.softmax(inp.logits.double(), dim=1).numpy()
    np.testing.assert_allclose(fwd["w"], np.take_along_axis(p, fwd["idx"].astype(np.int64), 1),
                               rtol=1e-12)
    zero = orc.layer_forward(inp.logits, inp.X, inp.W_gu, np.zeros_like(inp.W_d.float().numpy()), 4)
    assert (zero["Y"] == 0).all()


def test_token_forward_matches_layer_forward():
    inp = small_inputs(40, 16, 8, 2, 12, seed=10)
    fwd = orc.layer_forward(inp.logits, inp.X, inp.W_gu, inp.W_d, 2)
    toks = [0, 3, 17, 39]
    y = orc.token_forward(toks, fwd["idx"], fwd["w"], inp.X, inp.W_gu, inp.W_d)
    np.testing.assert_allclose(y, fwd["Y"][toks], rtol=1e-12, atol=1e-14)
