"""Pins of the oracle's backward against float64 autograd of a dense
formulation, central finite differences and invariants. CPU only."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as orc
from routed_grouped_gemm_router_b200.inputs import small_inputs


def dense_autograd(logits, X, W_gu, W_d, dY, k):
    """Dense float64 torch model: softmax over all experts, a 0/1 mask of the
    top-k set from ``torch.topk`` (held constant), renormalised weights, every
    expert applied to every token, weighted sum. Returns autograd gradients of
    <dY, Y>."""
    l = torch.tensor(np.asarray(logits, dtype=np.float64), requires_grad=True)
    x = torch.tensor(np.asarray(X, dtype=np.float64), requires_grad=True)
    wgu = torch.tensor(np.asarray(W_gu, dtype=np.float64), requires_grad=True)
    wd = torch.tensor(np.asarray(W_d, dtype=np.float64), requires_grad=True)
    I = wd.shape[2]
    p = torch.softmax(l, dim=1)
    mask = torch.zeros_like(p)
    mask.scatter_(1, torch.topk(l.detach(), k, dim=1).indices, 1.0)
    top = p * mask
    wdense = top / (top.sum(dim=1, keepdim=True) + 1e-20)
    g = torch.einsum("th,eih->tei", x, wgu[:, :I])
    u = torch.einsum("th,eih->tei", x, wgu[:, I:])
    o = torch.einsum("tei,ehi->teh", torch.nn.functional.silu(g) * u, wd)
    Y = torch.einsum("te,teh->th", wdense, o)
    (Y * torch.as_tensor(np.asarray(dY, dtype=np.float64))).sum().backward()
    return dict(Y=Y.detach().numpy(), dX=x.grad.numpy(), dW_gu=wgu.grad.numpy(),
                dW_d=wd.grad.numpy(), dlogits=l.grad.numpy())


@pytest.mark.parametrize("T,H,E,k,I,seed", [(6, 5, 4, 2, 3, 0), (9, 8, 6, 3, 4, 1),
                                            (5, 4, 3, 3, 2, 2), (7, 6, 5, 1, 3, 3)])
def test_backward_matches_dense_autograd(T, H, E, k, I, seed):
    inp = small_inputs(T, H, E, k, I, seed=seed)
    W_gu = inp.W_gu.float().numpy() * 25
    W_d = inp.W_d.float().numpy() * 25
    logits = inp.logits.numpy() * 4  # spread the routing weights
    fwd = orc.layer_forward(logits, inp.X, W_gu, W_d, k)
    bwd = orc.layer_backward(fwd, inp.dY, inp.X, W_gu, W_d, k)
    ref = dense_autograd(logits, inp.X.float().numpy(), W_gu, W_d, inp.dY.float().numpy(), k)
    np.testing.assert_allclose(fwd["Y"], ref["Y"], rtol=1e-10, atol=1e-12)
    for name in ("dX", "dW_gu", "dW_d", "dlogits"):
        np.testing.assert_allclose(bwd[name], ref[name], rtol=1e-9, atol=1e-11, err_msg=name)


def test_dlogits_central_differences():
    inp = small_inputs(4, 6, 5, 2, 4, seed=11)
    W_gu = inp.W_gu.float().numpy() * 25
    W_d = inp.W_d.float().numpy() * 25
    logits = (inp.logits.numpy() * 4).astype(np.float64)
    dY = inp.dY.float().numpy()
    fwd = orc.layer_forward(logits.astype(np.float32), inp.X, W_gu, W_d, 2)
    bwd = orc.layer_backward(fwd, dY, inp.X, W_gu, W_d, 2)
    # finite differences on a float64 copy of the routing chain, selection fixed
    idx = fwd["idx"]
    X = inp.X.float().numpy().astype(np.float64)

    def loss(lg):
        p = np.exp(lg - lg.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        top = np.take_along_axis(p, idx.astype(np.int64), 1)
        w = top / (top.sum(axis=1, keepdims=True) + 1e-20)
        total = 0.0
        for t in range(lg.shape[0]):
            for j in range(idx.shape[1]):
                _, _, _, o = orc.expert_mlp(X[t:t + 1], W_gu[idx[t, j]], W_d[idx[t, j]])
                total += w[t, j] * float((o[0] * dY[t]).sum())
        return total

    eps = 1e-6
    num = np.zeros_like(logits)
    for t in range(logits.shape[0]):
        for e in range(logits.shape[1]):
            lp = logits.copy(); lp[t, e] += eps
            lm = logits.copy(); lm[t, e] -= eps
            num[t, e] = (loss(lp) - loss(lm)) / (2 * eps)
    np.testing.assert_allclose(bwd["dlogits"], num, rtol=1e-5, atol=1e-7)


def test_dlogits_rows_sum_to_zero_and_empty_experts_get_zero_grads():
    inp = small_inputs(30, 8, 10, 2, 6, seed=12)
    logits = inp.logits.numpy().copy()
    logits[:, [2, 7]] -= 1e4   # experts 2 and 7 receive no tokens
    fwd = orc.layer_forward(logits, inp.X, inp.W_gu, inp.W_d, 2)
    bwd = orc.layer_backward(fwd, inp.dY, inp.X, inp.W_gu, inp.W_d, 2)
    assert fwd["counts"][2] == 0 and fwd["counts"][7] == 0
    np.testing.assert_allclose(bwd["dlogits"].sum(axis=1), 0.0, atol=1e-15)
    assert (bwd["dW_gu"][[2, 7]] == 0).all() and (bwd["dW_d"][[2, 7]] == 0).all()


def test_sampled_backward_matches_full():
    inp = small_inputs(48, 16, 8, 3, 12, seed=13)
    fwd = orc.layer_forward(inp.logits, inp.X, inp.W_gu, inp.W_d, 3)
    bwd = orc.layer_backward(fwd, inp.dY, inp.X, inp.W_gu, inp.W_d, 3)
    toks = [1, 5, 47]
    tb = orc.token_backward(toks, fwd["idx"], fwd["w"], fwd["probs"], inp.dY, inp.X, inp.W_gu, inp.W_d)
    np.testing.assert_allclose(tb["dX"], bwd["dX"][toks], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(tb["dlogits"], bwd["dlogits"][toks], rtol=1e-10, atol=1e-15)
    for e in (0, 4, 7):
        dgu, dd = orc.expert_weight_grads(e, fwd["offsets"], fwd["sorted_pair"], fwd["w"],
                                          inp.dY, inp.X, inp.W_gu, inp.W_d, 3)
        np.testing.assert_allclose(dgu, bwd["dW_gu"][e], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(dd, bwd["dW_d"][e], rtol=1e-12, atol=1e-14)
