"""Pins of the oracle's LoRA functions (adapters on the stacked expert
weights) against what fixes them independently: float64 autograd of a dense
model whose adapters are leaf tensors, central differences in the adapter
entries, the low-rank product evaluated without forming W + scale B A (per
token, unfused gate/up adapters, through the format conversion), and the
special case B = 0. CPU only."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as orc
from routed_grouped_gemm_router_b200.inputs import small_inputs
from routed_grouped_gemm_router_b200 import lora


def adapters(E, H, I, r, seed, mag=0.3):
    g = torch.Generator().manual_seed(seed)
    return dict(A_gu=(torch.randn(E, r, H, generator=g) * mag).double().numpy(),
                B_gu=(torch.randn(E, 2 * I, r, generator=g) * mag).double().numpy(),
                A_d=(torch.randn(E, r, I, generator=g) * mag).double().numpy(),
                B_d=(torch.randn(E, H, r, generator=g) * mag).double().numpy())


def dense_lora_autograd(logits, X, W_gu, W_d, dY, k, ad, scale):
    """Dense float64 torch model with the adapters as leaf tensors: every
    expert on every token, the adapter applied as x A^T then B^T (never as
    W + scale B A), top-k mask held constant. Autograd of <dY, Y>."""
    l = torch.tensor(np.asarray(logits, dtype=np.float64), requires_grad=True)
    x = torch.tensor(np.asarray(X, dtype=np.float64), requires_grad=True)
    wgu = torch.tensor(np.asarray(W_gu, dtype=np.float64))
    wd = torch.tensor(np.asarray(W_d, dtype=np.float64))
    A_gu, B_gu, A_d, B_d = (torch.tensor(ad[n], requires_grad=True) for n in ("A_gu", "B_gu", "A_d", "B_d"))
    I = wd.shape[2]
    p = torch.softmax(l, dim=1)
    mask = torch.zeros_like(p)
    mask.scatter_(1, torch.topk(l.detach(), k, dim=1).indices, 1.0)
    top = p * mask
    wdense = top / (top.sum(dim=1, keepdim=True) + 1e-20)
    gu = torch.einsum("th,eoh->teo", x, wgu) + scale * torch.einsum("ter,eor->teo",
                                                                     torch.einsum("th,erh->ter", x, A_gu), B_gu)
    g, u = gu[..., :I], gu[..., I:]
    h = torch.nn.functional.silu(g) * u
    o = torch.einsum("tei,ehi->teh", h, wd) + scale * torch.einsum("ter,ehr->teh",
                                                                   torch.einsum("tei,eri->ter", h, A_d), B_d)
    Y = torch.einsum("te,teh->th", wdense, o)
    (Y * torch.as_tensor(np.asarray(dY, dtype=np.float64))).sum().backward()
    return dict(Y=Y.detach().numpy(), dX=x.grad.numpy(), dlogits=l.grad.numpy(), dA_gu=A_gu.grad.numpy(),
                dB_gu=B_gu.grad.numpy(), dA_d=A_d.grad.numpy(), dB_d=B_d.grad.numpy())


CASES = [(6, 5, 4, 2, 3, 2, 0), (9, 8, 6, 3, 4, 3, 1), (7, 6, 5, 1, 3, 1, 2), (8, 8, 3, 3, 4, 4, 3)]


def _problem(T, H, E, k, I, r, seed):
    inp = small_inputs(T, H, E, k, I, seed=seed)
    W_gu = inp.W_gu.float().numpy() * 25
    W_d = inp.W_d.float().numpy() * 25
    logits = inp.logits.numpy() * 4
    return inp, W_gu, W_d, logits, adapters(E, H, I, r, seed + 100)


@pytest.mark.parametrize("T,H,E,k,I,r,seed", CASES)
def test_lora_matches_dense_autograd(T, H, E, k, I, r, seed):
    inp, W_gu, W_d, logits, ad = _problem(T, H, E, k, I, r, seed)
    scale = 1.7
    fwd = orc.lora_layer_forward(logits, inp.X, W_gu, W_d, k, ad["A_gu"], ad["B_gu"], ad["A_d"], ad["B_d"], scale)
    bwd = orc.lora_layer_backward(fwd, inp.dY, inp.X, k, ad["A_gu"], ad["B_gu"], ad["A_d"], ad["B_d"], scale)
    ref = dense_lora_autograd(logits, inp.X.float().numpy(), W_gu, W_d, inp.dY.float().numpy(), k, ad, scale)
    np.testing.assert_allclose(fwd["Y"], ref["Y"], rtol=1e-10, atol=1e-12)
    for name in ("dX", "dlogits", "dA_gu", "dB_gu", "dA_d", "dB_d"):
        np.testing.assert_allclose(bwd[name], ref[name], rtol=1e-9, atol=1e-11, err_msg=name)


def test_zero_B_is_the_base_layer():
    """B = 0 (the usual LoRA initialisation): the layer is the base layer,
    and dA = 0 since dA = scale B^T G."""
    inp, W_gu, W_d, logits, ad = _problem(8, 6, 4, 2, 5, 3, 7)
    ad["B_gu"][:] = 0.0
    ad["B_d"][:] = 0.0
    fwd = orc.lora_layer_forward(logits, inp.X, W_gu, W_d, 2, ad["A_gu"], ad["B_gu"], ad["A_d"], ad["B_d"], 2.0)
    base = orc.layer_forward(logits, inp.X, W_gu, W_d, 2)
    np.testing.assert_array_equal(fwd["Y"], base["Y"])
    bwd = orc.lora_layer_backward(fwd, inp.dY, inp.X, 2, ad["A_gu"], ad["B_gu"], ad["A_d"], ad["B_d"], 2.0)
    assert not bwd["dA_gu"].any() and not bwd["dA_d"].any()
    assert np.abs(bwd["dB_gu"]).max() > 0 and np.abs(bwd["dB_d"]).max() > 0


def test_adapter_central_differences():
    inp, W_gu, W_d, logits, ad = _problem(5, 4, 3, 2, 3, 2, 21)
    scale = 0.8
    dY = inp.dY.float().numpy().astype(np.float64)

    def loss(a):
        f = orc.lora_layer_forward(logits, inp.X, W_gu, W_d, 2, a["A_gu"], a["B_gu"], a["A_d"], a["B_d"], scale)
        return float((f["Y"] * dY).sum())

    fwd = orc.lora_layer_forward(logits, inp.X, W_gu, W_d, 2, ad["A_gu"], ad["B_gu"], ad["A_d"], ad["B_d"], scale)
    bwd = orc.lora_layer_backward(fwd, dY, inp.X, 2, ad["A_gu"], ad["B_gu"], ad["A_d"], ad["B_d"], scale)
    eps = 1e-6
    rng = np.random.default_rng(0)
    for name in ("A_gu", "B_gu", "A_d", "B_d"):
        for _ in range(6):
            ix = tuple(int(rng.integers(n)) for n in ad[name].shape)
            ap = {n: v.copy() for n, v in ad.items()}
            am = {n: v.copy() for n, v in ad.items()}
            ap[name][ix] += eps
            am[name][ix] -= eps
            num = (loss(ap) - loss(am)) / (2 * eps)
            assert abs(num - bwd["d" + name][ix]) <= 1e-6 * max(1.0, abs(num)), (name, ix, num, bwd["d" + name][ix])


def test_unfused_low_rank_per_token_equals_fused_oracle():
    """Gate and up adapters trained separately (unfused format), applied per
    token in low-rank form x A^T B^T, against the oracle on the fused adapter
    that ``lora.fuse_gate_up`` builds from them; and the reverse conversion."""
    T, H, E, k, I, r = 7, 6, 4, 2, 5, 3
    inp, W_gu, W_d, logits, ad = _problem(T, H, E, k, I, r, 31)
    g = torch.Generator().manual_seed(5)
    A_g, A_u = torch.randn(E, r, H, generator=g).double(), torch.randn(E, 2, H, generator=g).double()
    B_g, B_u = torch.randn(E, I, r, generator=g).double(), torch.randn(E, I, 2, generator=g).double()
    A_gu, B_gu = lora.fuse_gate_up(A_g, B_g, A_u, B_u)
    assert A_gu.shape == (E, r + 2, H) and B_gu.shape == (E, 2 * I, r + 2)
    scale = 1.3
    fwd = orc.lora_layer_forward(logits, inp.X, W_gu, W_d, k, A_gu.numpy(), B_gu.numpy(), ad["A_d"], ad["B_d"], scale)
    X = inp.X.double().numpy()
    idx, w, _ = orc.route(logits, k)
    Y = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            x = X[t]
            gg = W_gu[e, :I] @ x + scale * (B_g[e].numpy() @ (A_g[e].numpy() @ x))
            uu = W_gu[e, I:] @ x + scale * (B_u[e].numpy() @ (A_u[e].numpy() @ x))
            hh = gg / (1.0 + np.exp(-gg)) * uu
            o = W_d[e] @ hh + scale * (ad["B_d"][e] @ (ad["A_d"][e] @ hh))
            Y[t] += w[t, j] * o
    np.testing.assert_allclose(fwd["Y"], Y, rtol=1e-10, atol=1e-12)
    # back to the unfused format: each projection keeps its rows of B_gu A_gu
    a1, b1, a2, b2 = lora.unfuse_gate_up(A_gu, B_gu)
    np.testing.assert_array_equal((b1 @ a1).numpy(), (B_gu @ A_gu).numpy()[:, :I])
    np.testing.assert_array_equal((b2 @ a2).numpy(), (B_gu @ A_gu).numpy()[:, I:])


def test_planted_mistakes_fail_the_autograd_pin(monkeypatch):
    """A dropped scale in the adapter gradients, or B used untransposed in
    dA, must each fail the dense-autograd pin."""
    T, H, E, k, I, r, seed = CASES[1]
    inp, W_gu, W_d, logits, ad = _problem(T, H, E, k, I, r, seed)
    ref = dense_lora_autograd(logits, inp.X.float().numpy(), W_gu, W_d, inp.dY.float().numpy(), k, ad, 1.7)
    orig = orc.lora_layer_backward

    def no_scale(fwd, dY, X, k, A_gu, B_gu, A_d, B_d, scale):
        return orig(fwd, dY, X, k, A_gu, B_gu, A_d, B_d, 1.0)

    def b_untransposed(fwd, dY, X, k, A_gu, B_gu, A_d, B_d, scale):
        g = orig(fwd, dY, X, k, A_gu, B_gu, A_d, B_d, scale)
        g["dA_gu"] = scale * np.einsum("eor,eoi->eri", np.ascontiguousarray(B_gu[:, ::-1]), g["dW_gu"])
        return g

    for bad in (no_scale, b_untransposed):
        monkeypatch.setattr(orc, "lora_layer_backward", bad)
        fwd = orc.lora_layer_forward(logits, inp.X, W_gu, W_d, k, ad["A_gu"], ad["B_gu"], ad["A_d"], ad["B_d"], 1.7)
        bwd = orc.lora_layer_backward(fwd, inp.dY, inp.X, k, ad["A_gu"], ad["B_gu"], ad["A_d"], ad["B_d"], 1.7)
        assert not np.allclose(bwd["dA_gu"], ref["dA_gu"], rtol=1e-6, atol=1e-9), bad.__name__
    monkeypatch.setattr(orc, "lora_layer_backward", orig)
