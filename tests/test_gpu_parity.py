"""CUDA path (through the C ABI) against the CPU oracle, element by element,
on seeded inputs that span several tiles, ragged tails and the degenerate
cases of the method. Routing/permutation must be bit-exact; floating outputs
within max|err| <= 2e-2 * max|ref|."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as orc
from routed_grouped_gemm_router_b200.inputs import WORKLOADS, make_inputs, small_inputs

import gpu_util as U

pytestmark = pytest.mark.gpu

# (T, H, E, k, I): several M/N/K tiles, tails in every dimension, E not a
# power of two, k = 1 and k = E, one row, rows < one tile.
SHAPES = [
    (256, 128, 8, 2, 256),     # the tiny layer
    (300, 200, 6, 2, 136),     # ragged H and I (not multiples of 64)
    (700, 320, 13, 3, 192),    # E not a power of two, N tails at 256
    (64, 256, 4, 4, 64),       # k = E (weights = softmax)
    (96, 128, 16, 1, 128),     # k = 1 (weight = 1)
    (1, 64, 4, 2, 64),         # a single token
    (3, 72, 5, 2, 40),         # fewer rows than one tile, tiny tails
    (1200, 512, 32, 4, 384),   # 32 experts of about 150 rows (one pair tile or a tail each)
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "T%d_H%d_E%d_k%d_I%d" % s)
def test_layer_matches_oracle(shape):
    """The default path (permuted copies Xp / dYp) against the oracle, and the
    gather-fused path bit for bit against it."""
    T, H, E, k, I = shape
    inp = small_inputs(T, H, E, k, I, seed=sum(shape))
    st, grads = U.run_layer(inp, k)
    st_g, grads_g = U.run_layer(inp, k, gather=True)
    U.assert_same_results(st_g, grads_g, st, grads)
    fwd, bwd = U.oracle_full(inp, k)
    U.check_routing_exact(st, fwd)
    U.assert_rel(U.to_np(st.h), fwd["h"], "h")
    U.assert_rel(U.to_np(st.gu)[:, :I], fwd["g"], "g")
    U.assert_rel(U.to_np(st.gu)[:, I:], fwd["u"], "u")
    U.assert_rel(U.to_np(st.O), fwd["O"], "O")
    U.assert_rel(U.to_np(st.Y), fwd["Y"], "Y")
    U.assert_rel(U.to_np(grads["dX"]), bwd["dX"], "dX")
    U.assert_rel(U.to_np(grads["dW_gu"]), bwd["dW_gu"], "dW_gu")
    U.assert_rel(U.to_np(grads["dW_d"]), bwd["dW_d"], "dW_d")
    U.assert_rel(U.to_np(grads["dlogits"]), bwd["dlogits"], "dlogits")


def test_one_expert_spans_many_pair_tiles():
    """Expert 0 is in every token's top-k: its segment is 2148 rows, eight
    256-row pair tiles and a 100-row tail (the one-CTA tail tiles); the other
    three experts share the second slot (about 716 rows each: two pair tiles
    and a tail of more than 128 rows). Every stored intermediate (g, u, h, O)
    and every output and gradient element by element against the oracle."""
    T, H, E, k, I = 2148, 256, 4, 2, 320
    inp = small_inputs(T, H, E, k, I, seed=11)
    logits = inp.logits.clone()
    logits[:, 0] += 30.0
    inp.logits = logits.contiguous()
    st, grads = U.run_layer(inp, k)
    fwd, bwd = U.oracle_full(inp, k)
    U.check_routing_exact(st, fwd)
    assert fwd["counts"][0] == T and fwd["counts"][1:].min() > 512 + 128
    U.assert_rel(U.to_np(st.gu)[:, :I], fwd["g"], "g")
    U.assert_rel(U.to_np(st.gu)[:, I:], fwd["u"], "u")
    U.assert_rel(U.to_np(st.h), fwd["h"], "h")
    U.assert_rel(U.to_np(st.O), fwd["O"], "O")
    U.assert_rel(U.to_np(st.Y), fwd["Y"], "Y")
    for name in ("dX", "dW_gu", "dW_d", "dlogits"):
        U.assert_rel(U.to_np(grads[name]), bwd[name], name)
    # expert 0's rows alone (the segment that spans the most tiles)
    lo, hi = fwd["offsets"][0], fwd["offsets"][1]
    U.assert_rel(U.to_np(st.O)[lo:hi], fwd["O"][lo:hi], "O[expert 0]")
    U.assert_rel(U.to_np(grads["dW_gu"])[0], bwd["dW_gu"][0], "dW_gu[expert 0]")


def test_empty_experts_and_one_hot_expert():
    """20 of 24 experts dead (no rows, dW exactly 0); one expert in every token."""
    T, H, E, k, I = 400, 128, 24, 3, 128
    inp = small_inputs(T, H, E, k, I, seed=5)
    logits = inp.logits.clone()
    logits[:, 4:] -= 1e4
    logits[:, 2] += 30.0            # expert 2 receives every token
    inp.logits = logits.contiguous()
    st, grads = U.run_layer(inp, k)
    fwd, bwd = U.oracle_full(inp, k)
    U.check_routing_exact(st, fwd)
    assert fwd["counts"][2] == T and (fwd["counts"][4:] == 0).all()
    U.assert_rel(U.to_np(st.Y), fwd["Y"], "Y")
    for name in ("dX", "dW_gu", "dW_d", "dlogits"):
        U.assert_rel(U.to_np(grads[name]), bwd[name], name)
    assert (U.to_np(grads["dW_gu"])[4:] == 0).all() and (U.to_np(grads["dW_d"])[4:] == 0).all()


def test_adversarial_routing_ties():
    """Exact ties, all-equal rows and signed zeros: ids must follow the
    lower-index rule bit-exactly."""
    T, E, k = 512, 37, 5
    g = torch.Generator().manual_seed(3)
    vals = torch.tensor([-1.0, -0.0, 0.0, 0.5, 2.0, -1e4])
    logits = vals[torch.randint(0, len(vals), (T, E), generator=g)].contiguous()
    logits[0] = 0.25
    from routed_grouped_gemm_router_b200 import binding as B
    idx, w, probs = B.moe_route(logits.cuda(), k)
    ridx, rw, rp = orc.route(logits.numpy(), k)
    assert (idx.cpu().numpy() == ridx).all()
    np.testing.assert_allclose(w.cpu().numpy(), rw, atol=U.W_ABS_TOL, rtol=0)
    perm = B.moe_permute(idx, E)
    c, o, sp, pp = orc.permute(ridx, E)
    assert (perm["counts"].cpu().numpy() == c).all() and (perm["offsets"].cpu().numpy() == o).all()
    assert (perm["sorted_pair"].cpu().numpy() == sp).all() and (perm["pair_pos"].cpu().numpy() == pp).all()


@pytest.mark.parametrize("E", [1, 33, 1000, 1024])
def test_route_permute_wide_and_narrow_E(E):
    T = 2048 if E < 1000 else 300
    k = min(E, 8)
    g = torch.Generator().manual_seed(E)
    logits = torch.randn(T, E, generator=g)
    from routed_grouped_gemm_router_b200 import binding as B
    idx, w, probs = B.moe_route(logits.cuda(), k)
    ridx, rw, rp = orc.route(logits.numpy(), k)
    assert (idx.cpu().numpy() == ridx).all()
    np.testing.assert_allclose(w.cpu().numpy(), rw, atol=U.W_ABS_TOL, rtol=0)
    np.testing.assert_allclose(probs.cpu().numpy(), rp, atol=1e-6, rtol=1e-4)
    perm = B.moe_permute(idx, E)
    c, o, sp, pp = orc.permute(ridx, E)
    assert (perm["sorted_pair"].cpu().numpy() == sp).all() and (perm["pair_pos"].cpu().numpy() == pp).all()
    assert (perm["counts"].cpu().numpy() == c).all()


@pytest.mark.parametrize("gather", [True, False])
def test_recompute_gate_up_when_not_saved(gather):
    T, H, E, k, I = 500, 256, 8, 2, 192
    inp = small_inputs(T, H, E, k, I, seed=21)
    st, grads = U.run_layer(inp, k, save_gu=False, gather=gather)
    fwd, bwd = U.oracle_full(inp, k)
    assert st.gu is None
    for name in ("dX", "dW_gu", "dW_d", "dlogits"):
        U.assert_rel(U.to_np(grads[name]), bwd[name], name)


def test_non_default_stream():
    T, H, E, k, I = 256, 128, 8, 2, 256
    inp = small_inputs(T, H, E, k, I, seed=0)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        st, grads = U.run_layer(inp, k, stream=s)
    s.synchronize()
    fwd, bwd = U.oracle_full(inp, k)
    U.assert_rel(U.to_np(st.Y), fwd["Y"], "Y")
    U.assert_rel(U.to_np(grads["dX"]), bwd["dX"], "dX")


@pytest.mark.parametrize("gather", [True, False])
def test_empty_batch(gather):
    from routed_grouped_gemm_router_b200 import binding as B
    from routed_grouped_gemm_router_b200 import layer
    E, k, H, I = 8, 2, 64, 64
    logits = torch.empty(0, E, device="cuda")
    X = torch.empty(0, H, dtype=torch.bfloat16, device="cuda")
    W_gu = torch.randn(E, 2 * I, H, device="cuda").bfloat16()
    W_d = torch.randn(E, H, I, device="cuda").bfloat16()
    st = layer.forward(logits, X, W_gu, W_d, k, gather=gather)
    assert st.Y.shape == (0, H) and (st.perm["counts"] == 0).all() and (st.perm["offsets"] == 0).all()
    grads = layer.backward(st, torch.empty(0, H, dtype=torch.bfloat16, device="cuda"), W_gu, W_d)
    assert (grads["dW_gu"] == 0).all() and (grads["dW_d"] == 0).all()
    assert B.last_device_status() == 0


def test_repeated_calls_are_deterministic():
    T, H, E, k, I = 1000, 256, 16, 4, 256
    inp = small_inputs(T, H, E, k, I, seed=9)
    a, ga = U.run_layer(inp, k)
    b, gb = U.run_layer(inp, k)
    assert torch.equal(a.Y, b.Y) and torch.equal(ga["dX"], gb["dX"])
    assert torch.equal(ga["dW_gu"], gb["dW_gu"]) and torch.equal(ga["dlogits"], gb["dlogits"])


def test_backward_without_h():
    """The backward recomputes h from g|u; passing no h gives the same gradients."""
    from routed_grouped_gemm_router_b200 import binding as B
    T, H, E, k, I = 600, 192, 10, 3, 160
    inp = small_inputs(T, H, E, k, I, seed=31)
    st, grads = U.run_layer(inp, k)
    d = U.to_dev(inp)
    p = st.perm
    g2 = B.moe_layer_bwd(d["dY"], p["Xp"], st.gu, None, st.probs, st.topk_idx, st.topk_w, p["offsets"],
                         p["sorted_pair"], p["pair_pos"], T, E, k, d["W_gu"], d["W_d"])
    for name in ("dX", "dW_gu", "dW_d", "dlogits"):
        assert torch.equal(g2[name], grads[name]), name
