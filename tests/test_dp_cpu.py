"""Data-parallel partitioning of the layer, on the CPU with two gloo ranks.

Each rank runs the oracle on its own token shard (the weights replicated),
lays its weight gradients out in the package's flat gradient buffer and sums
them with the package's exchange (all-reduce, or reduce-scatter). The result
must be the full batch's weight gradient, and the per-token results (Y, dX,
d logits) of each shard must be the full batch's rows: the layer has no
coupling between tokens except through the weight-gradient sums."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import moe_oracle as orc
from routed_grouped_gemm_router_b200 import dp
from routed_grouped_gemm_router_b200.inputs import small_inputs

SHAPE = (97, 64, 6, 2, 48)  # T odd: the shards differ in size


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shard_inputs(inp, lo, hi):
    import copy
    s = copy.copy(inp)
    s.X, s.logits, s.dY = inp.X[lo:hi].contiguous(), inp.logits[lo:hi].contiguous(), inp.dY[lo:hi].contiguous()
    return s


def _rank_main(rank, world, port, op, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T, H, E, k, I = SHAPE
        inp = small_inputs(T, H, E, k, I, seed=7)    # the same batch and weights on every rank
        lo, hi = dp.token_shard(T, world, rank)
        s = _shard_inputs(inp, lo, hi)
        fwd = orc.layer_forward(s.logits, s.X, s.W_gu, s.W_d, k)
        bwd = orc.layer_backward(fwd, s.dY, s.X, s.W_gu, s.W_d, k)
        flat, views = dp.flat_weight_grads(E, H, I, dtype=torch.float64)
        views["dW_gu"].copy_(torch.from_numpy(bwd["dW_gu"]))
        views["dW_d"].copy_(torch.from_numpy(bwd["dW_d"]))
        piece = dp.sync_weight_grads(flat, op=op)
        out[rank] = dict(lo=lo, hi=hi, flat=flat.numpy().copy(),
                         piece=None if piece is None else piece.numpy().copy(),
                         Y=fwd["Y"], dX=bwd["dX"], dlogits=bwd["dlogits"], idx=fwd["idx"])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("op", ["allreduce", "reduce_scatter"])
def test_token_sharded_layer_sums_to_the_full_batch(op):
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), op, out), nprocs=world, join=True)
    T, H, E, k, I = SHAPE
    inp = small_inputs(T, H, E, k, I, seed=7)
    fwd = orc.layer_forward(inp.logits, inp.X, inp.W_gu, inp.W_d, k)
    bwd = orc.layer_backward(fwd, inp.dY, inp.X, inp.W_gu, inp.W_d, k)
    full = np.concatenate([bwd["dW_gu"].ravel(), bwd["dW_d"].ravel()])
    assert [(out[r]["lo"], out[r]["hi"]) for r in range(world)] == [(0, 49), (49, 97)]
    for r in range(world):
        o = out[r]
        lo, hi = o["lo"], o["hi"]
        assert (o["idx"] == fwd["idx"][lo:hi]).all()      # routing is per token
        for name, ref in (("Y", fwd["Y"]), ("dX", bwd["dX"]), ("dlogits", bwd["dlogits"])):
            np.testing.assert_allclose(o[name], ref[lo:hi], rtol=1e-12, atol=1e-14, err_msg=name)
        if op == "allreduce":
            np.testing.assert_allclose(o["flat"], full, rtol=1e-12, atol=1e-14)
        else:
            per = -(-full.size // world)
            ref = np.zeros(per * world)
            ref[:full.size] = full
            np.testing.assert_allclose(o["piece"], ref[r * per:(r + 1) * per], rtol=1e-12, atol=1e-14)
    if op == "reduce_scatter":  # the exchange leaves the local gradient as it was: a shard's part only
        assert not np.allclose(out[0]["flat"], full)


def test_token_shard_partitions():
    for T in (0, 1, 7, 97, 16384):
        for world in (1, 2, 3, 8):
            spans = [dp.token_shard(T, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == T
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    with pytest.raises(ValueError):
        dp.token_shard(10, 2, 2)


def test_flat_grad_views_share_one_buffer():
    E, H, I = 3, 16, 8
    flat, v = dp.flat_weight_grads(E, H, I, router=True)
    assert v["dW_gu"].shape == (E, 2 * I, H) and v["dW_d"].shape == (E, H, I) and v["dW_r"].dtype == torch.float32
    assert v["dW_gu"].data_ptr() == flat.data_ptr()
    assert v["dW_d"].data_ptr() == flat.data_ptr() + E * 2 * I * H * flat.element_size()
    assert v["dW_d"].data_ptr() % 16 == 0 and v["dW_gu"].is_contiguous() and v["dW_d"].is_contiguous()
    flat.zero_()
    v["dW_d"].fill_(1)
    assert float(flat.float().sum()) == E * H * I
