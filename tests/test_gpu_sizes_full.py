"""Full-size layers in the launch configuration the benchmark times: routing
and permutation checked in full (bit-exact), outputs and gradients checked on
seeded samples the oracle computes one token / one expert at a time."""
import numpy as np
import pytest

from oracle import moe_oracle as orc
from routed_grouped_gemm_router_b200.inputs import WORKLOADS, make_inputs

import gpu_util as U

pytestmark = pytest.mark.gpu


def _sample_tokens(T, n, seed):
    rng = np.random.default_rng(seed)
    pick = rng.choice(T, size=min(n, T), replace=False).tolist()
    return sorted(set(pick + [0, T - 1]))


def _sample_experts(counts):
    live = np.nonzero(counts)[0]
    picks = {int(live[0]), int(live[-1]), int(np.argmax(counts)), int(live[np.argmin(counts[live])])}
    dead = np.nonzero(counts == 0)[0]
    if dead.size:
        picks.add(int(dead[0]))
    return sorted(picks)


@pytest.mark.parametrize("name", ["qwen3-30b-a3b", "gpt-oss-20b", "qwen3-235b-a22b", "zipf-t64", "zipf-t32768"])
def test_full_size_layer(name):
    wl = WORKLOADS[name]
    k = wl.k
    inp = make_inputs(wl, seed=0, with_dy=True)
    st, grads = U.run_layer(inp, k)
    idx, w, probs = orc.route(inp.logits, k)
    counts, offsets, sorted_pair, pair_pos = orc.permute(idx, wl.E)
    U.check_routing_exact(st, dict(idx=idx, w=w, probs=probs, counts=counts, offsets=offsets,
                                   sorted_pair=sorted_pair, pair_pos=pair_pos))
    toks = _sample_tokens(wl.T, 48, seed=1)
    y_ref = orc.token_forward(toks, idx, w, inp.X, inp.W_gu, inp.W_d)
    U.assert_rel(U.to_np(st.Y[toks]), y_ref, f"{name} Y")
    tb = orc.token_backward(toks, idx, w, probs, inp.dY, inp.X, inp.W_gu, inp.W_d)
    U.assert_rel(U.to_np(grads["dX"][toks]), tb["dX"], f"{name} dX")
    U.assert_rel(U.to_np(grads["dlogits"][toks]), tb["dlogits"], f"{name} dlogits")
    for e in _sample_experts(counts):
        dgu, dd = orc.expert_weight_grads(e, offsets, sorted_pair, w, inp.dY, inp.X, inp.W_gu, inp.W_d, k)
        if counts[e] == 0:
            assert (U.to_np(grads["dW_gu"][e]) == 0).all() and (U.to_np(grads["dW_d"][e]) == 0).all()
        else:
            U.assert_rel(U.to_np(grads["dW_gu"][e]), dgu, f"{name} dW_gu[{e}]")
            U.assert_rel(U.to_np(grads["dW_d"][e]), dd, f"{name} dW_d[{e}]")


@pytest.mark.parametrize("name", ["qwen3-30b-a3b", "zipf-t32768", "zipf-t64"])
def test_full_size_gathered_equals_permuted(name):
    """At full size (long weight-gradient K for the hot experts, 20 empty
    experts), the gathered operand loads give bit-identical results to the
    loads from the permuted copies."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl, seed=0, with_dy=True)
    a, ga = U.run_layer(inp, wl.k, gather=True)
    b, gb = U.run_layer(inp, wl.k)
    U.assert_same_results(a, ga, b, gb)
