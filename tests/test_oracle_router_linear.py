"""Pins of the oracle's router Linear (logits = X W_r^T) and its backward:
closed forms, float64 autograd of the dense layer with the router inside it,
and central differences on W_r. CPU only."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as orc
from routed_grouped_gemm_router_b200.inputs import small_inputs


def test_identity_router_selects_hidden_features():
    """W_r = the first E rows of the identity: logits are X's first E features."""
    rng = np.random.default_rng(0)
    X = rng.standard_normal((7, 12))
    W_r = np.eye(12)[:5]
    np.testing.assert_array_equal(orc.router_logits(X, W_r), X[:, :5])


def test_rank_one_closed_form():
    """X = a b^T and W_r = c d^T give logits = (b.d) a c^T."""
    a, b, c, d = (np.arange(1.0, n + 1) for n in (4, 6, 3, 6))
    X, W_r = np.outer(a, b), np.outer(c, d)
    np.testing.assert_allclose(orc.router_logits(X, W_r), (b @ d) * np.outer(a, c), rtol=1e-15)


def test_backward_closed_form_single_token():
    """One token, one expert: dW_r = dl * x, dX = dl * w."""
    x = np.array([[1.0, -2.0, 3.0]])
    w = np.array([[0.5, 0.25, -1.0]])
    dW, dX = orc.router_logits_backward(np.array([[2.0]]), x, w)
    np.testing.assert_array_equal(dW, 2.0 * x)
    np.testing.assert_array_equal(dX, 2.0 * w)


def dense_block_autograd(X, W_r, W_gu, W_d, dY, k):
    """Dense float64 torch model of the whole block: logits = X W_r^T, softmax,
    0/1 top-k mask from torch.topk (held constant), renormalised weights, every
    expert on every token, weighted sum. Autograd gradients of <dY, Y>; X gets
    gradient through both the router and the experts."""
    x = torch.tensor(np.asarray(X, dtype=np.float64), requires_grad=True)
    wr = torch.tensor(np.asarray(W_r, dtype=np.float64), requires_grad=True)
    wgu = torch.tensor(np.asarray(W_gu, dtype=np.float64))
    wd = torch.tensor(np.asarray(W_d, dtype=np.float64))
    I = wd.shape[2]
    l = torch.nn.functional.linear(x, wr)
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
    return dict(logits=l.detach().numpy(), Y=Y.detach().numpy(), dX=x.grad.numpy(), dW_r=wr.grad.numpy())


def oracle_block(X, W_r, W_gu, W_d, dY, k):
    logits = orc.router_logits(X, W_r)
    fwd = orc.layer_forward(logits, X, W_gu, W_d, k)
    bwd = orc.layer_backward(fwd, dY, X, W_gu, W_d, k)
    dW_r, dX_router = orc.router_logits_backward(bwd["dlogits"], X, W_r)
    return logits, fwd, bwd, dW_r, bwd["dX"] + dX_router


@pytest.mark.parametrize("T,H,E,k,I,seed", [(6, 5, 4, 2, 3, 0), (9, 8, 6, 3, 4, 1), (5, 7, 3, 1, 2, 2)])
def test_block_gradients_match_dense_autograd(T, H, E, k, I, seed):
    inp = small_inputs(T, H, E, k, I, seed=seed)
    X = inp.X.float().numpy().astype(np.float64)
    W_r = inp.W_r.numpy().astype(np.float64) * 40  # spread the routing weights
    W_gu = inp.W_gu.float().numpy() * 25
    W_d = inp.W_d.float().numpy() * 25
    dY = inp.dY.float().numpy()
    logits, fwd, bwd, dW_r, dX = oracle_block(X, W_r, W_gu, W_d, dY, k)
    ref = dense_block_autograd(X, W_r, W_gu, W_d, dY, k)
    np.testing.assert_allclose(logits, ref["logits"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(fwd["Y"], ref["Y"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dW_r, ref["dW_r"], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dX, ref["dX"], rtol=1e-9, atol=1e-11)


def test_dW_r_central_differences():
    """<dY, Y> differentiated numerically in W_r (selection fixed by the
    unperturbed logits; the steps are far too small to change it)."""
    T, H, E, k, I = 4, 6, 5, 2, 3
    inp = small_inputs(T, H, E, k, I, seed=7)
    X = inp.X.float().numpy().astype(np.float64)
    W_r = inp.W_r.numpy().astype(np.float64) * 40
    W_gu = inp.W_gu.float().numpy() * 25
    W_d = inp.W_d.float().numpy() * 25
    dY = inp.dY.float().numpy()
    _, fwd, _, dW_r, _ = oracle_block(X, W_r, W_gu, W_d, dY, k)
    idx = fwd["idx"]

    def loss(wr):
        f = orc.layer_forward(orc.router_logits(X, wr), X, W_gu, W_d, k)
        assert (f["idx"] == idx).all()
        return float((f["Y"] * dY).sum())

    eps = 1e-6
    num = np.zeros_like(W_r)
    for e in range(E):
        for h in range(H):
            wp = W_r.copy(); wp[e, h] += eps
            wm = W_r.copy(); wm[e, h] -= eps
            num[e, h] = (loss(wp) - loss(wm)) / (2 * eps)
    np.testing.assert_allclose(dW_r, num, rtol=1e-5, atol=1e-7)


def test_mutated_router_backward_fails_pins():
    """A transposed operand in the router's dX (W_r^T in place of W_r on a
    square case) is caught by the dense-autograd pin."""
    T, H, E, k, I = 6, 4, 4, 2, 3
    inp = small_inputs(T, H, E, k, I, seed=3)
    X = inp.X.float().numpy().astype(np.float64)
    W_r = inp.W_r.numpy().astype(np.float64) * 40
    W_gu = inp.W_gu.float().numpy() * 25
    W_d = inp.W_d.float().numpy() * 25
    dY = inp.dY.float().numpy()
    _, fwd, bwd, _, _ = oracle_block(X, W_r, W_gu, W_d, dY, k)
    wrong = bwd["dX"] + bwd["dlogits"] @ W_r.T
    ref = dense_block_autograd(X, W_r, W_gu, W_d, dY, k)
    assert not np.allclose(wrong, ref["dX"], rtol=1e-6, atol=1e-9)
