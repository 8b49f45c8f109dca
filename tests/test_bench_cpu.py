"""The bench's own bookkeeping, on the CPU: the roofline bound and work of
each kernel, the DRAM traffic read from the committed ncu summaries (scaled
from a reduced capture where one stands in for the full layer), the oracle
sample's expert cut, and the configuration labels."""
import argparse

import bench
from routed_grouped_gemm_router_b200.inputs import WORKLOADS, make_inputs

PEAKS = {"hbm_gbs": 6548.2, "bf16_tflops": 1642.8, "bf16_tflops_sustained": 1402.8}


def test_dgrad_down_bound_follows_the_workload():
    kind30, work30 = bench.kernel_work("gemm_bwd_dgrad_down", WORKLOADS["qwen3-30b-a3b"], 0, PEAKS)
    kind235, work235 = bench.kernel_work("gemm_bwd_dgrad_down", WORKLOADS["qwen3-235b-a22b"], 0, PEAKS)
    wl = WORKLOADS["qwen3-235b-a22b"]
    assert kind30 == "hbm" and kind235 == "tensor"
    assert work235 == 2.0 * wl.H * wl.I * wl.P
    # without peaks the byte count is kept, as before
    assert bench.kernel_work("gemm_bwd_dgrad_down", wl)[0] == "hbm"
    assert bench.kernel_work("gemm_fwd_gate_up", wl)[1] == 4.0 * wl.H * wl.I * wl.P


def test_decode_sized_batch_is_hbm_bound():
    """64 tokens: the expert GEMMs stream the active experts' weights, so each
    takes the HBM bound with those bytes; the big layers keep the tensor bound."""
    wl = WORKLOADS["zipf-t64"]
    names = ("gemm_fwd_gate_up", "gemm_fwd_down", "gemm_bwd_dgrad_gate_up", "gemm_bwd_dgrad_down",
             "gemm_bwd_wgrad_gate_up", "gemm_bwd_wgrad_down")
    for name in names:
        kind, work = bench.kernel_work(name, wl, 0, PEAKS, active=90)
        assert kind == "hbm", name
        assert work == bench.gemm_bytes(name, wl, 0, 90)
    H, I, P, E = wl.H, wl.I, wl.P, wl.E
    # gate/up forward: X rows in, the 90 experts' [W_g; W_u] in, h and g|u out
    assert bench.gemm_bytes("gemm_fwd_gate_up", wl, 0, 90) == P * H * 2 + 90 * 2 * I * H * 2 + P * I * 2 + P * 4 * I
    # the weight gradient writes every expert's block, idle ones included
    assert bench.gemm_bytes("gemm_bwd_wgrad_down", wl, 0, 90) == P * H * 2 + P * I * 2 + E * H * I * 2
    for wname in ("qwen3-235b-a22b", "gpt-oss-20b"):
        for name in names:
            assert bench.kernel_work(name, WORKLOADS[wname], 0, PEAKS)[0] == "tensor", (wname, name)
    assert bench.gemm_bytes("gather_x", wl) is None


def test_traffic_from_committed_summaries():
    t235, src235 = bench.measured_traffic("gemm_bwd_wgrad_gate_up", "qwen3-235b-a22b")
    t16, src16 = bench.measured_traffic("gemm_bwd_wgrad_gate_up", "qwen3-235b-a22b-e16-t2048")
    assert t16 is not None and src16.endswith(".txt")
    assert t235 == 8 * t16 and "(x8)" in src235         # scaled by the units processed
    t30, src30 = bench.measured_traffic("gemm_bwd_wgrad_gate_up", "qwen3-30b-a3b")
    assert t30 is not None and "(x" not in src30        # the workload's own capture, as it stands
    assert bench.measured_traffic("gemm_bwd_wgrad_gate_up", "gpt-oss-20b") == (None, None)
    assert bench.measured_traffic("no_such_kernel", "qwen3-235b-a22b") == (None, None)


def test_source_hash_covers_each_kernels_files():
    assert bench.kernel_source_sha("router_bwd") != bench.kernel_source_sha("route_hist")
    assert bench.kernel_source_sha("gemm_fwd_down") == bench.kernel_source_sha("gemm_bwd_wgrad_gate_up")


def test_cpu_sample_cuts_experts_and_tokens():
    wl = WORKLOADS["tiny"]
    inp = make_inputs(wl, seed=0)
    sample, ts, es, lo = bench.cpu_sample(inp, wl, target_s=0.01)
    assert es == wl.E and lo is None
    assert sample.X.shape[0] == ts and sample.logits.shape == (ts, es)
    wl2 = type(wl)("cut", 40, 64, 40, 2, 32)
    inp2 = make_inputs(wl2, seed=1)
    s2, ts2, es2, _ = bench.cpu_sample(inp2, wl2, target_s=0.01)
    assert es2 == 16 and s2.W_gu.shape[0] == 16 and s2.W_d.shape[0] == 16 and s2.logits.shape[1] == 16
    assert "first 16 of 40 experts" in bench.sample_desc(wl2, ts2, es2)


def test_config_labels():
    wl = WORKLOADS["qwen3-235b-a22b"]
    base = dict(router_linear=False, gather_fused=False, cuda_graph=False, dw_f32=False, lora=0, seed=0)
    one = bench.workload_config(wl, argparse.Namespace(gpus=1, **base))
    assert one["parallelism"] == "single GPU" and "qwen3-235b-a22b MoE layer fwd+bwd" in one["workload"]
    dp8 = bench.workload_config(wl, argparse.Namespace(gpus=8, grad_sync="allreduce", **base))
    assert dp8["parallelism"].startswith("dp8")
    ep8 = bench.workload_config(wl, argparse.Namespace(gpus=8, ep=True, **base))
    assert ep8["parallelism"].startswith("ep8")
    rep = bench.workload_config(wl, argparse.Namespace(gpus=4, grad_sync="none", **base))
    assert rep["parallelism"] == "replicas x4"
    assert bench.aggregate_tflops(2, 1e12, 10, 1000.0) == 20.0


def test_datasheet_fractions():
    """The datasheet denominators sit beside the measured ones: 2.25 PFLOP/s
    dense bf16 for a tensor-bound kernel, 8 TB/s for an HBM-bound one."""
    assert bench.datasheet_fracs({"bound": "tensor", "achieved": 1125.0}) == (2250.0, 0.5)
    assert bench.datasheet_fracs({"bound": "hbm", "achieved": 6000.0}) == (8000.0, 0.75)
    assert bench.datasheet_fracs({"bound": "alu", "achieved": 1.0}) == (None, None)


def test_routing_stats():
    even = bench.routing_stats([4, 4, 4, 4])
    assert even == {"max_rows": 4, "empty_experts": 0, "mean_rows": 4.0, "gini": 0.0}
    one = bench.routing_stats([0, 0, 0, 12])
    assert one["max_rows"] == 12 and one["empty_experts"] == 3 and abs(one["gini"] - 0.75) < 1e-12
    # brute force: mean absolute difference over all pairs / (2 * mean)
    c = [3, 0, 7, 1, 9]
    mad = sum(abs(a - b) for a in c for b in c) / len(c) ** 2
    assert abs(bench.routing_stats(c)["gini"] - mad / (2 * sum(c) / len(c))) < 1e-12
