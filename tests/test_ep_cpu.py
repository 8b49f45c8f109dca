"""Expert-parallel plumbing on the CPU with two gloo ranks.

Each rank has its own tokens and owns half of the experts. The rows travel
to their experts' owners and back through ep.ep_forward / ep.ep_backward,
with the oracle standing in for the CUDA steps (ep_util.OracleOps). Every
rank's Y, dX and d logits must equal the whole layer's on its tokens, and
the weight gradients of its experts must equal the whole layer's over both
ranks' tokens together: the exchange must neither lose, duplicate nor
misplace a row."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import moe_oracle as orc
from routed_grouped_gemm_router_b200 import ep
from routed_grouped_gemm_router_b200.inputs import small_inputs

import ep_util

CASES = {
    "balanced": dict(T=(37, 50), H=48, E=8, k=3, I=40, bias=None),
    # rank 1's experts are never chosen: it receives no rows at all
    "idle_owner": dict(T=(20, 33), H=32, E=8, k=2, I=24, bias="low_half"),
}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_inputs(case, rank):
    c = CASES[case]
    inp = small_inputs(c["T"][rank], c["H"], c["E"], c["k"], c["I"], seed=100 + rank)
    W = small_inputs(4, c["H"], c["E"], c["k"], c["I"], seed=7)  # the same expert weights on every rank
    logits = inp.logits.clone()
    if c["bias"] == "low_half":
        logits[:, c["E"] // 2:] -= 1e4
    return logits, inp.X, inp.dY, W.W_gu, W.W_d


def _rank_main(rank, world, port, case, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c = CASES[case]
        E, k = c["E"], c["k"]
        logits, X, dY, W_gu, W_d = _rank_inputs(case, rank)
        lo, hi = ep.experts_of_rank(E, world, rank)
        ops = ep_util.OracleOps()
        st = ep.ep_forward(logits, X.double(), W_gu[lo:hi], W_d[lo:hi], k, E, ops=ops)
        g = ep.ep_backward(st, dY.double(), W_gu[lo:hi], W_d[lo:hi], ops=ops)
        out[rank] = dict(Y=st.Y.numpy(), dX=g["dX"].numpy(), dlogits=g["dlogits"].numpy(),
                         dW_gu=g["dW_gu"].numpy(), dW_d=g["dW_d"].numpy(), P_recv=st.P_recv,
                         send=st.send_counts, recv=st.recv_counts)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", sorted(CASES))
def test_expert_parallel_equals_the_whole_layer(case):
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), case, out), nprocs=world, join=True)
    c = CASES[case]
    E, k = c["E"], c["k"]
    per_rank = [_rank_inputs(case, r) for r in range(world)]
    # per-token results: the whole layer on each rank's own tokens
    for r in range(world):
        logits, X, dY, W_gu, W_d = per_rank[r]
        fwd = orc.layer_forward(logits, X, W_gu, W_d, k)
        bwd = orc.layer_backward(fwd, dY, X, W_gu, W_d, k)
        np.testing.assert_allclose(out[r]["Y"], fwd["Y"], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(out[r]["dX"], bwd["dX"], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(out[r]["dlogits"], bwd["dlogits"], rtol=1e-10, atol=1e-13)
    # weight gradients: the whole layer over both ranks' tokens, this rank's experts
    logits = torch.cat([p[0] for p in per_rank])
    X = torch.cat([p[1] for p in per_rank])
    dY = torch.cat([p[2] for p in per_rank])
    W_gu, W_d = per_rank[0][3], per_rank[0][4]
    fwd = orc.layer_forward(logits, X, W_gu, W_d, k)
    bwd = orc.layer_backward(fwd, dY, X, W_gu, W_d, k)
    for r in range(world):
        lo, hi = ep.experts_of_rank(E, world, r)
        np.testing.assert_allclose(out[r]["dW_gu"], bwd["dW_gu"][lo:hi], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(out[r]["dW_d"], bwd["dW_d"][lo:hi], rtol=1e-10, atol=1e-12)
    # the exchange's bookkeeping: what one rank sends the other receives
    assert out[0]["send"][1] == out[1]["recv"][0] and out[1]["send"][0] == out[0]["recv"][1]
    assert sum(out[0]["send"]) == c["T"][0] * k and sum(out[1]["send"]) == c["T"][1] * k
    if case == "idle_owner":
        assert out[1]["P_recv"] == 0


def test_experts_of_rank():
    assert ep.experts_of_rank(128, 8, 3) == (48, 64)
    assert ep.experts_of_rank(8, 1, 0) == (0, 8)
    with pytest.raises(ValueError):
        ep.experts_of_rank(10, 4, 0)
