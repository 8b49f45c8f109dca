"""Plants plausible mistakes in the oracle (on the CPU, through monkeypatch)
and checks that the pins catch each one: a pin that cannot fail pins nothing."""
import numpy as np
import pytest

from oracle import moe_oracle as orc
import test_oracle_backward as tb
import test_oracle_forward as tf
import test_oracle_permute as tp
import test_oracle_route as tr


def _no_renorm(logits, k):
    probs = orc.softmax(logits)
    idx = orc.select_topk(logits, k)
    return idx, np.take_along_axis(probs, idx.astype(np.int64), 1), probs


def _high_index_wins(logits, k):
    l = np.asarray(logits, dtype=np.float32)
    T, E = l.shape
    return np.lexsort((-np.broadcast_to(np.arange(E), (T, E)), -l), axis=1)[:, :k].astype(np.int32)


def _swap_gate_up(x, W_gu_e, W_d_e):
    I = W_d_e.shape[1]
    return _orig_mlp(x, np.concatenate([W_gu_e[I:], W_gu_e[:I]]), W_d_e)


def _sigmoid_gate(x, W_gu_e, W_d_e):
    I = W_d_e.shape[1]
    g = x @ W_gu_e[:I].T
    u = x @ W_gu_e[I:].T
    h = orc.sigmoid(g) * u
    return g, u, h, h @ W_d_e.T


def _unstable_permute(idx, E):
    counts, offsets, sp, pp = _orig_permute(idx, E)
    for e in range(E):
        sp[offsets[e]:offsets[e + 1]] = sp[offsets[e]:offsets[e + 1]][::-1]
    pp[sp] = np.arange(sp.size, dtype=np.int32)
    return counts, offsets, sp, pp


def _router_bwd_sign(dw, w, probs, idx):
    return _orig_router_bwd(dw, -w, probs, idx)


def _combine_wrong_index(O, pair_pos, T, k):
    return _orig_combine(O, np.argsort(pair_pos), T, k)


_orig_mlp = orc.expert_mlp
_orig_permute = orc.permute
_orig_router_bwd = orc.router_backward
_orig_combine = orc.combine


CASES = [
    ("route", _no_renorm, lambda: tr.test_route_closed_form(tr._golden_cases()[0])),
    ("select_topk", _high_index_wins, lambda: tr.test_selection_matches_rank_count(0)),
    ("expert_mlp", _swap_gate_up, lambda: tf.test_forward_matches_dense_bruteforce(5, 4, 3, 2, 3, 0)),
    ("expert_mlp", _sigmoid_gate, lambda: tf.test_forward_matches_dense_bruteforce(5, 4, 3, 2, 3, 0)),
    ("permute", _unstable_permute, lambda: tp.test_permute_matches_bruteforce(64, 8, 2, 2)),
    ("router_backward", _router_bwd_sign, lambda: tb.test_backward_matches_dense_autograd(6, 5, 4, 2, 3, 0)),
    ("combine", _combine_wrong_index, lambda: tf.test_forward_matches_dense_bruteforce(6, 3, 4, 1, 2, 1)),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}:{c[1].__name__}" for c in CASES])
def test_planted_mistake_is_caught(case, monkeypatch):
    name, bad, pin = case
    monkeypatch.setattr(orc, name, bad)
    with pytest.raises(AssertionError):
        pin()


def test_planted_silu_derivative_mistake_is_caught(monkeypatch):
    """dg without the (1 + g(1 - s)) factor of silu' must fail the autograd pin."""
    real = orc.layer_backward

    def wrong_backward(fwd, dY, X, W_gu, W_d, k):
        fwd2 = dict(fwd)
        out = real(fwd2, dY, X, W_gu, W_d, k)
        # recompute dW_gu's gate half and dX with dg = dh * u * s only
        Xf = orc._f64(X); dYf = orc._f64(dY)
        W_gu = orc._f64(W_gu); W_d = orc._f64(W_d)
        I = W_d.shape[2]
        dX = np.zeros_like(out["dX"])
        for e in range(W_gu.shape[0]):
            lo, hi = int(fwd["offsets"][e]), int(fwd["offsets"][e + 1])
            if lo == hi:
                continue
            q = fwd["sorted_pair"][lo:hi]; tok = q // k
            g, u = fwd["g"][lo:hi], fwd["u"][lo:hi]
            dh = (fwd["w"].reshape(-1)[q, None] * dYf[tok]) @ W_d[e]
            s = orc.sigmoid(g)
            dg = dh * u * s
            du = dh * g * s
            dX[tok] += dg @ W_gu[e, :I] + du @ W_gu[e, I:]
        out["dX"] = dX
        return out

    monkeypatch.setattr(orc, "layer_backward", wrong_backward)
    with pytest.raises(AssertionError):
        tb.test_backward_matches_dense_autograd(6, 5, 4, 2, 3, 0)
