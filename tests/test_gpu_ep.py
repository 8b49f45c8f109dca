"""The expert-parallel layer on a GPU: two processes each own half of the
experts and their own tokens, and run every step through the C ABI
(ep.ep_forward / ep.ep_backward with the CUDA ops). The rows cross between
the processes through gloo (this pool gives one GPU; the two processes'
kernels never wait on each other).

Each rank's Y, dX and d logits must match the oracle's whole layer on its
tokens, and its experts' weight gradients the oracle's over both ranks'
tokens, within the layer's tolerance. They must also match the local
(single-process) CUDA layer on the same tokens: routing bit for bit, the
rest within the tolerance."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import moe_oracle as orc
from routed_grouped_gemm_router_b200.inputs import small_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "balanced": dict(T=(600, 733), H=256, E=8, k=2, I=192, bias=None),
    "idle_owner": dict(T=(300, 257), H=128, E=8, k=3, I=128, bias="low_half"),
}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_inputs(case, rank):
    c = CASES[case]
    inp = small_inputs(c["T"][rank], c["H"], c["E"], c["k"], c["I"], seed=200 + rank)
    W = small_inputs(4, c["H"], c["E"], c["k"], c["I"], seed=9)
    logits = inp.logits.clone()
    if c["bias"] == "low_half":
        logits[:, c["E"] // 2:] -= 1e4
    return logits.contiguous(), inp.X, inp.dY, W.W_gu, W.W_d


def _rank_main(rank, world, port, case, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from routed_grouped_gemm_router_b200 import binding as B
        from routed_grouped_gemm_router_b200 import ep, layer
        torch.cuda.set_device(0)
        c = CASES[case]
        E, k = c["E"], c["k"]
        logits, X, dY, W_gu, W_d = (t.cuda() for t in _rank_inputs(case, rank))
        lo, hi = ep.experts_of_rank(E, world, rank)
        W_gu_l, W_d_l = W_gu[lo:hi].contiguous(), W_d[lo:hi].contiguous()
        st = ep.ep_forward(logits, X, W_gu_l, W_d_l, k, E)
        g = ep.ep_backward(st, dY, W_gu_l, W_d_l)
        loc = layer.forward(logits, X, W_gu, W_d, k)
        gl = layer.backward(loc, dY, W_gu, W_d)
        assert B.last_device_status() == 0
        f = lambda t: t.float().cpu().numpy()
        out[rank] = dict(Y=f(st.Y), dX=f(g["dX"]), dlogits=f(g["dlogits"]), dW_gu=f(g["dW_gu"]),
                         dW_d=f(g["dW_d"]), P_recv=st.P_recv, idx_same=bool(torch.equal(st.idx, loc.topk_idx)),
                         Y_loc=f(loc.Y), dX_loc=f(gl["dX"]), dlogits_loc=f(gl["dlogits"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", sorted(CASES))
def test_expert_parallel_layer_on_gpu(case):
    import gpu_util as U
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), case, out), nprocs=world, join=True,
                       start_method="spawn")
    c = CASES[case]
    E, k = c["E"], c["k"]
    per_rank = [_rank_inputs(case, r) for r in range(world)]
    for r in range(world):
        o = out[r]
        logits, X, dY, W_gu, W_d = per_rank[r]
        fwd = orc.layer_forward(logits, X, W_gu, W_d, k)
        bwd = orc.layer_backward(fwd, dY, X, W_gu, W_d, k)
        assert o["idx_same"], "routing differs from the local layer"
        U.assert_rel(o["Y"], fwd["Y"], f"rank {r} Y")
        U.assert_rel(o["dX"], bwd["dX"], f"rank {r} dX")
        U.assert_rel(o["dlogits"], bwd["dlogits"], f"rank {r} dlogits")
        U.assert_rel(o["Y"], o["Y_loc"], f"rank {r} Y vs the local layer")
        U.assert_rel(o["dX"], o["dX_loc"], f"rank {r} dX vs the local layer")
        U.assert_rel(o["dlogits"], o["dlogits_loc"], f"rank {r} dlogits vs the local layer")
    logits = torch.cat([p[0] for p in per_rank])
    X = torch.cat([p[1] for p in per_rank])
    dY = torch.cat([p[2] for p in per_rank])
    W_gu, W_d = per_rank[0][3], per_rank[0][4]
    fwd = orc.layer_forward(logits, X, W_gu, W_d, k)
    bwd = orc.layer_backward(fwd, dY, X, W_gu, W_d, k)
    for r in range(world):
        lo, hi = (r * E // world, (r + 1) * E // world)
        if np.abs(bwd["dW_gu"][lo:hi]).max() == 0:  # experts that no token chose: exactly zero
            assert (out[r]["dW_gu"] == 0).all() and (out[r]["dW_d"] == 0).all()
        else:
            U.assert_rel(out[r]["dW_gu"], bwd["dW_gu"][lo:hi], f"rank {r} dW_gu")
            U.assert_rel(out[r]["dW_d"], bwd["dW_d"][lo:hi], f"rank {r} dW_d")
    if case == "idle_owner":
        assert out[1]["P_recv"] == 0


@pytest.mark.parametrize("shape", [(700, 320, 13, 3, 192), (96, 128, 16, 1, 128), (1, 64, 4, 2, 64)],
                         ids=lambda s: "T%d_H%d_E%d_k%d_I%d" % s)
def test_ep_calls_match_the_layer_calls(shape):
    """moe_layer_bwd_pair_dw gives moe_layer_bwd's dX and dW bit for bit and
    the oracle's per-pair routing-weight gradients; moe_router_bwd_from_dw on
    those (per sorted row) gives moe_layer_bwd's d logits; moe_ep_pack_rows
    gives each sorted row's owner-local expert and weight."""
    import gpu_util as U
    from routed_grouped_gemm_router_b200 import binding as B
    T, H, E, k, I = shape
    inp = small_inputs(T, H, E, k, I, seed=sum(shape) + 1)
    st, grads = U.run_layer(inp, k)
    d = U.to_dev(inp)
    p = st.perm
    g = B.moe_layer_bwd_pair_dw(d["dY"], p["Xp"], st.gu, st.h, st.topk_w, p["offsets"], p["sorted_pair"],
                                p["pair_pos"], T, E, k, d["W_gu"], d["W_d"])
    for name in ("dX", "dW_gu", "dW_d"):
        assert torch.equal(g[name], grads[name]), name
    fwd, bwd = U.oracle_full(inp, k)
    U.assert_rel(U.to_np(g["dw"]).reshape(T, k), bwd["dw"], "dw")
    dw_rows = torch.empty_like(g["dw"])
    dw_rows[p["pair_pos"].long()] = g["dw"]          # per pair -> per sorted row
    dl = B.moe_router_bwd_from_dw(dw_rows, p["pair_pos"], st.probs, st.topk_idx, st.topk_w)
    U.assert_rel(U.to_np(dl), U.to_np(grads["dlogits"]), "dlogits from dw vs the layer's")
    U.assert_rel(U.to_np(dl), bwd["dlogits"], "dlogits from dw vs the oracle")
    E_l = E if E % 2 else E // 2
    le, rw = B.moe_ep_pack_rows(p["offsets"], p["sorted_pair"], st.topk_w, T, E, k, E_l)
    off = p["offsets"].cpu().numpy()
    want = np.concatenate([np.full(off[e + 1] - off[e], e % E_l) for e in range(E)])
    assert (le.cpu().numpy() == want).all()
    assert torch.equal(rw, st.topk_w.reshape(-1)[p["sorted_pair"].long()])
    assert B.last_device_status() == 0
