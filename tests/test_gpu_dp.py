"""The data-parallel step on a GPU: two processes, each running the CUDA
layer (through the C ABI) on its own half of one batch with the same
weights, sum their weight gradients with the package's exchange (gloo here:
this pool gives one GPU, and the two processes' kernels never wait on each
other). The summed gradients must match the oracle's full-batch gradients
within the layer's tolerance, and each half's outputs the full batch's rows."""
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

SHAPE = (601, 256, 12, 3, 192)  # T odd: the halves differ in size


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from routed_grouped_gemm_router_b200 import binding as B
        from routed_grouped_gemm_router_b200 import dp, layer
        torch.cuda.set_device(0)
        T, H, E, k, I = SHAPE
        inp = small_inputs(T, H, E, k, I, seed=21)
        lo, hi = dp.token_shard(T, world, rank)
        dev = "cuda:0"
        X, logits, dY = (t[lo:hi].contiguous().to(dev) for t in (inp.X, inp.logits, inp.dY))
        W_gu, W_d = inp.W_gu.to(dev), inp.W_d.to(dev)
        flat, views = dp.flat_weight_grads(E, H, I, dtype=torch.bfloat16, device=dev)
        bufs = layer.allocate(hi - lo, E, k, H, I, dev)
        bufs["grads"].update(views)
        st = layer.forward(logits, X, W_gu, W_d, k, bufs=bufs)
        g = layer.backward(st, dY, W_gu, W_d, bufs=bufs)
        assert g["dW_gu"].data_ptr() == flat.data_ptr()
        assert B.last_device_status() == 0
        summed = flat.float().cpu()                   # gloo sums on the host
        dp.sync_weight_grads(summed, op="allreduce")
        out[rank] = dict(lo=lo, hi=hi, flat=summed.numpy(), Y=st.Y.float().cpu().numpy(),
                         dX=g["dX"].float().cpu().numpy(), dlogits=g["dlogits"].cpu().numpy())
    finally:
        dist.destroy_process_group()


def test_two_process_layer_gradients_sum_to_the_full_batch():
    import gpu_util as U
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    T, H, E, k, I = SHAPE
    inp = small_inputs(T, H, E, k, I, seed=21)
    fwd, bwd = U.oracle_full(inp, k)
    n_gu = E * 2 * I * H
    for r in range(world):
        o = out[r]
        U.assert_rel(o["flat"][:n_gu].reshape(E, 2 * I, H), bwd["dW_gu"], f"rank {r} summed dW_gu")
        U.assert_rel(o["flat"][n_gu:].reshape(E, H, I), bwd["dW_d"], f"rank {r} summed dW_d")
        lo, hi = o["lo"], o["hi"]
        U.assert_rel(o["Y"], fwd["Y"][lo:hi], f"rank {r} Y")
        U.assert_rel(o["dX"], bwd["dX"][lo:hi], f"rank {r} dX")
        U.assert_rel(o["dlogits"], bwd["dlogits"][lo:hi], f"rank {r} dlogits")
    assert np.array_equal(out[0]["flat"], out[1]["flat"]), "the ranks must hold the same summed gradient"
