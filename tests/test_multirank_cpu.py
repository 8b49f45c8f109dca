"""The benchmark's N > 1 path on the CPU: two gloo ranks, each with its own
seeded batch, take the max of their device-timed milliseconds and report the
whole-job throughput (weak scaling, no data-path collective)."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from routed_grouped_gemm_router_b200.inputs import make_inputs, WORKLOADS


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    w, r, lr = bench.world_info()
    assert (w, r, lr) == (world, rank, rank)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = WORKLOADS["tiny"]
        inp = make_inputs(wl, seed=0 + rank)          # every rank its own batch
        my_ms = [10.0 + rank, 20.0 - rank]            # stand-in per-rank device times
        mx = bench.max_over_ranks(my_ms, "cpu")
        out[rank] = (mx, float(inp.X.float().sum()))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == [11.0, 20.0]
    assert out[0][1] != out[1][1], "ranks must draw different batches"
    wl = WORKLOADS["tiny"]
    f = bench.step_flops(wl)
    # two ranks, 5 steps each, slowest rank 11 ms in total
    assert abs(bench.aggregate_tflops(2, f, 5, 11.0) - 2 * f * 5 / 0.011 / 1e12) < 1e-12
