#!/usr/bin/env python
"""Benchmark of the fused MoE expert layer (forward + backward) on B200.

One step = the whole layer: moe_route -> moe_permute -> moe_experts_fwd ->
moe_combine -> moe_layer_bwd on one synthetic batch already resident in HBM.
Prints ONE JSON line (rank 0). Default workload: the Qwen3-235B-A22B-shaped
layer (T=16384, H=4096, E=128, k=8, I=1536), forward and backward.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle on a bounded sample

With N > 1 (launched by torch.distributed.run) every rank runs the layer on
its own batch (weak scaling) and the ranks' weight gradients are summed over
NCCL after every backward (--grad-sync allreduce | reduce_scatter | none); the
time is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import glob
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from routed_grouped_gemm_router_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "MoE layer fwd/bwd TFLOP/s and tokens/s on 1 B200; % of bf16 tensor peak"
UNIT = "TFLOP/s"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# Algorithmic work per launch of each kernel, as a function of the workload:
# GEMMs in flops (bf16 tensor cores), memory kernels in bytes (HBM). A kernel
# with both significant flops and bytes (dgrad through down) is reported
# against whichever roofline bounds it on this workload (`peaks` given).
def gemm_bytes(name, wl, lora_r=0, active=None):
    """Algorithmic bytes of one expert GEMM call of the layer (with g|u saved
    in the forward): each operand row read once, the weights of the experts
    that have rows (``active``; all E when not given) read once, each output
    written once. The weight gradients write all E experts (zeros for idle
    ones). None for kernels that are not expert GEMMs."""
    T, H, E, k, I, P = wl.T, wl.H, wl.E, wl.k, wl.I, wl.P
    r = lora_r
    Ea = E if active is None else active
    w_gu, w_d = Ea * 2 * I * H * 2, Ea * H * I * 2
    # with adapters the row-grouped GEMMs also read Z (P r) and B (r N per expert)
    z = (lambda n: P * r * 2 + Ea * r * n * 2) if r else (lambda n: 0)
    part = P * 2 * ((I + 255) // 256) * 4          # routing-weight partials of the dgrad through down
    table = {
        "gemm_fwd_gate_up": P * H * 2 + w_gu + P * I * 2 + P * 2 * I * 2 + z(2 * I),
        "gemm_recompute_gate_up": P * H * 2 + w_gu + P * 2 * I * 2 + z(2 * I),
        "gemm_fwd_down": P * I * 2 + w_d + P * 4 + P * H * 2 + z(H),
        # dYp, W_d and g|u read; dGU, w*h and the partials written
        "gemm_bwd_dgrad_down": P * H * 2 + w_d + P * 2 * I * 2 + P * 2 * I * 2 + P * I * 2 + part + z(I),
        "gemm_bwd_dgrad_gate_up": P * 2 * I * 2 + w_gu + P * H * 2 + z(H),
        "gemm_bwd_wgrad_gate_up": P * H * 2 + P * 2 * I * 2 + E * 2 * I * H * 2,
        "gemm_bwd_wgrad_down": P * H * 2 + P * I * 2 + E * H * I * 2,
    }
    return table.get(name)


def kernel_work(name, wl, lora_r=0, peaks=None, active=None):
    """(bound, work) of one launch of kernel ``name``: FLOPs for a tensor-bound
    kernel, bytes for an HBM-bound one. With ``peaks`` an expert GEMM takes the
    bound whose time at the measured peak is the longer (a decode-sized batch
    streams the active experts' weights and is HBM-bound)."""
    T, H, E, k, I, P = wl.T, wl.H, wl.E, wl.k, wl.I, wl.P
    r = lora_r
    flops = {
        # with adapters of rank r the row-grouped GEMMs also run the adapter
        # term as r more K columns ([act | Z] [W | B])
        "gemm_fwd_gate_up": 4.0 * H * I * P + 4.0 * I * r * P, "gemm_fwd_down": 2.0 * H * I * P + 2.0 * H * r * P,
        "gemm_recompute_gate_up": 4.0 * H * I * P + 4.0 * I * r * P,
        "gemm_bwd_dgrad_gate_up": 4.0 * H * I * P + 2.0 * H * r * P,
        "gemm_bwd_wgrad_gate_up": 4.0 * H * I * P, "gemm_bwd_wgrad_down": 2.0 * H * I * P,
        # adapter products (useful flops; their tiles are 256 wide in r)
        "gemm_lora_z_gate_up": 2.0 * H * r * P, "gemm_lora_z_down": 2.0 * I * r * P,
        "gemm_lora_v_down": 2.0 * H * r * P, "gemm_lora_v_gate_up": 4.0 * I * r * P,
        "gemm_lora_da_gate_up": 2.0 * H * r * P, "gemm_lora_db_gate_up": 4.0 * I * r * P,
        "gemm_lora_da_down": 2.0 * I * r * P, "gemm_lora_db_down": 2.0 * H * r * P,
    }
    if name in flops:
        gb = gemm_bytes(name, wl, r, active)
        if peaks is not None and gb is not None and \
                gb / (peaks["hbm_gbs"] * 1e9) > flops[name] / (peaks["bf16_tflops"] * 1e12):
            return "hbm", float(gb)
        return "tensor", flops[name]
    nbytes = {
        # one read of each source row (L2 serves the k re-reads), one write per pair row
        "gather_x": T * H * 2 + P * H * 2 + P * 4, "gather_dy": T * H * 2 + P * H * 2 + P * 4,
        "combine_y": P * H * 2 + T * H * 2 + P * 4, "combine_dx": P * H * 2 + T * H * 2 + P * 4,
        "route": T * E * 4 * 2 + T * k * 8,
        "router_bwd": T * E * 4 * 2 + T * k * 12 + P * 8 * ((I + 255) // 256),
        "permute_count": P * 4, "permute_scan": E * 8, "permute_scatter": P * 12,
        # routing with the per-chunk expert counts (one byte per expert, rounded up to 16, per 32 tokens),
        # then the scan-and-scatter kernel that reads those counts and the ids once and writes the permutation
        "route_hist": T * E * 4 * 2 + T * k * 8 + -(-T // 32) * (-(-E // 16) * 16),
        "permute_scan_scatter": -(-T // 32) * (-(-E // 16) * 16) + P * 4 + P * 8 + E * 8,
        # router Linear: X (bf16) and W_r (fp32) read once, logits / dW_r / dX written once
        "router_split_w": E * H * 4 + 3 * E * H * 2, "router_split_dlogits": T * E * 4 + 3 * T * E * 2,
        "gemm_router_logits": T * H * 2 + E * H * 4 + T * E * 4,
        "gemm_router_wgrad": T * H * 2 + T * E * 4 + E * H * 4, "router_sum_splits": 2 * E * H * 4,
        "gemm_router_dgrad": T * E * 4 + E * H * 4 + 2 * T * H * 2,
        "lora_weight_rows": 2 * P * r * 2 + P * 8,
        # dgrad through down: HBM-bound on the narrower layers (its bytes at the
        # measured copy bandwidth take longer than its flops at the bf16 peak)
        "gemm_bwd_dgrad_down": gemm_bytes("gemm_bwd_dgrad_down", wl, r, active),
    }
    if name == "gemm_bwd_dgrad_down" and peaks is not None:
        # dYp W_d per pair: 2 H I flops (plus the adapter's 2 H r)
        fl = 2.0 * H * I * P + 2.0 * H * r * P
        if fl / (peaks["bf16_tflops"] * 1e12) > nbytes[name] / (peaks["hbm_gbs"] * 1e9):
            return "tensor", fl
    return "hbm", float(nbytes.get(name, 0))


# Datasheet figures per B200, reported beside the measured denominators: dense
# bf16 tensor throughput (without 2:4 sparsity) and HBM3e bandwidth.
DATASHEET_PEAKS = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}


def datasheet_fracs(roof):
    """The roofline's achieved rate against the datasheet peak of its bound
    (None for a bound the datasheet does not cover)."""
    key = {"tensor": "bf16_tflops", "hbm": "hbm_gbs"}.get(roof["bound"])
    if key is None:
        return None, None
    return DATASHEET_PEAKS[key], roof["achieved"] / DATASHEET_PEAKS[key]


def routing_stats(counts):
    """The realised expert histogram of a batch (rows per expert): largest
    segment, experts with no rows, mean rows per expert and the Gini
    coefficient of the row counts (0 = every expert the same, (E-1)/E = one
    expert takes every row)."""
    c = sorted(int(x) for x in counts)
    n, tot = len(c), sum(c)
    gini = 0.0 if tot == 0 else 2.0 * sum((i + 1) * x for i, x in enumerate(c)) / (n * tot) - (n + 1) / n
    return {"max_rows": c[-1] if c else 0, "empty_experts": sum(1 for x in c if x == 0),
            "mean_rows": tot / n if n else 0.0, "gini": gini}


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# Device-code files behind each kernel (the launch code in moe_lib.cu is not
# part of a kernel's identity).
_KERNEL_FILES = [
    (("gemm_router_", "router_split_", "router_sum_"), ["router_linear.cuh"]),
    (("gemm_",), ["grouped_gemm.cuh"]),
    (("router_bwd",), ["router_bwd.cuh"]),  # before "route", which it starts with
    (("route",), ["route.cuh"]),
    (("permute_", "gather_"), ["permute.cuh"]),
    (("combine_",), ["combine.cuh"]),
]


def kernel_source_sha(kernel=None):
    """Hash of the device code of `kernel` (its own file plus the shared
    sm100.cuh / common.cuh), or of every source file when kernel is None."""
    csrc = os.path.join(ROOT, "routed_grouped_gemm_router_b200", "csrc")
    files = sorted(glob.glob(os.path.join(csrc, "*")))
    if kernel is not None:
        for prefixes, own in _KERNEL_FILES:
            if kernel.startswith(prefixes):
                files = [os.path.join(csrc, f) for f in own + ["sm100.cuh", "common.cuh"]]
                break
    h = hashlib.sha256()
    for p in files:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary of the same kernel
    source, and the summary's file name; (None, None) when there is none or
    the sources changed since.

    A summary of the workload itself is used as it stands. A summary of a
    scaled case (fewer experts and tokens, the same rows per expert and the
    same H, I, k) names the workload it stands for (`scales_to:`) and the
    ratio of units processed (`scale_factor:`, full-size pairs over the
    case's pairs); its per-launch traffic is multiplied by that ratio, since
    every operand the kernel moves (expert weights, expert rows) grows in
    proportion to the experts and pairs."""
    sha = kernel_source_sha(kernel)
    direct, scaled = None, None
    for p in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.txt"))):
        text = open(p).read()
        if not (re.search(rf"^kernel: {re.escape(kernel)}$", text, re.M)
                and re.search(rf"^source_sha: {sha}$", text, re.M)):
            continue
        m = re.search(r"^traffic_bytes_per_launch: ([0-9.eE+]+)$", text, re.M)
        if not m:
            continue
        if re.search(rf"^workload: {re.escape(workload)}$", text, re.M):
            direct = (float(m.group(1)), os.path.basename(p))
        elif re.search(rf"^scales_to: {re.escape(workload)}$", text, re.M):
            f = re.search(r"^scale_factor: ([0-9.eE+]+)$", text, re.M)
            if f:
                scaled = (float(m.group(1)) * float(f.group(1)), os.path.basename(p) + f" (x{f.group(1)})")
    return direct or scaled or (None, None)


class ClockSampler:
    """SM clock, power and clock-event reasons sampled about every 2 ms
    (NVML, read-only) inside the timed window."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.rows = []
        self.active = False
        self.stop_flag = False
        self.thread = None
        self.nvml = None

    def start(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nvml = nv
            try:  # the CUDA device by UUID (CUDA and NVML may number devices differently)
                uuid = "GPU-" + str(torch.cuda.get_device_properties(self.idx).uuid)
                self.handle = nv.nvmlDeviceGetHandleByUUID(uuid.encode())
            except Exception:
                self.handle = nv.nvmlDeviceGetHandleByIndex(self.idx)
        except Exception:
            self.nvml = None
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def window(self, on):
        self.active = on

    def _run(self):
        nv = self.nvml
        mx = None
        n = 0
        pw = 0.0
        while not self.stop_flag:
            if self.active and nv is not None:
                try:
                    if mx is None:  # static: read once
                        mx = nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM)
                    sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                    if n % 4 == 0:  # power is an averaged reading: every 4th sample
                        pw = nv.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
                    n += 1
                    self.rows.append((sm, mx, pw, rs))
                except Exception:
                    pass
            time.sleep(0.002)

    def stop(self):
        self.stop_flag = True
        if self.thread is not None:
            self.thread.join(timeout=2)
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [r[0] for r in self.rows]
        reasons = sorted({n for r in self.rows for n, bit in self.REASONS.items() if r[3] & bit})
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": max(r[1] for r in self.rows),
                "reasons": reasons, "samples": len(self.rows), "power_w_max": max(r[2] for r in self.rows),
                "power_w_median": statistics.median([r[2] for r in self.rows]), "source": "NVML, ~2 ms"}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_step(inp_sub, k, backward, router=False, lora=None):
    from oracle import moe_oracle as orc
    logits = orc.router_logits(inp_sub.X, inp_sub.W_r) if router else inp_sub.logits
    if lora is not None:
        a = [lora[n] for n in ("A_gu", "B_gu", "A_d", "B_d")] + [lora["scale"]]
        fwd = orc.lora_layer_forward(logits, inp_sub.X, inp_sub.W_gu, inp_sub.W_d, k, *a)
        if backward:
            orc.lora_layer_backward(fwd, inp_sub.dY, inp_sub.X, k, *a)
        return
    fwd = orc.layer_forward(logits, inp_sub.X, inp_sub.W_gu, inp_sub.W_d, k)
    if backward:
        bwd = orc.layer_backward(fwd, inp_sub.dY, inp_sub.X, inp_sub.W_gu, inp_sub.W_d, k)
        if router:
            orc.router_logits_backward(bwd["dlogits"], inp_sub.X, inp_sub.W_r)


CPU_SAMPLE_EXPERTS = 16


def cpu_sample(inp, wl, target_s, router=False, lora=None):
    """A bounded sample of the batch for the oracle: the first T_s tokens
    routed over the first E_s = min(E, 16) experts (the logits, router weight
    and expert weights cut to those experts), T_s sized so one oracle step
    takes about target_s seconds on the host cores. The oracle widens every
    expert weight it is given to float64 on each call, so the expert cut keeps
    that fixed cost (and the host memory) bounded on the large layers; the
    per-expert problem (H, I, k) is the workload's own. Returns the sample,
    T_s, E_s and the sample's adapters (or None)."""
    import copy

    es = min(wl.E, max(CPU_SAMPLE_EXPERTS, 2 * wl.k))
    lo = None
    if lora is not None:
        lo = {n: (v[:es] if n != "scale" else v) for n, v in lora.items()}

    def sub(ts):
        s = copy.copy(inp)
        s.X = inp.X[:ts].contiguous()
        s.logits = inp.logits[:ts, :es].contiguous()
        s.W_r = inp.W_r[:es].contiguous()
        s.W_gu, s.W_d = inp.W_gu[:es].contiguous(), inp.W_d[:es].contiguous()
        s.dY = inp.dY[:ts].contiguous() if inp.dY is not None else None
        return s

    ts = min(wl.T, 64)
    t0 = time.perf_counter()
    oracle_step(sub(ts), wl.k, wl.backward, router, lo)
    dt = time.perf_counter() - t0
    while ts < wl.T and dt < target_s / 4:
        ts = min(wl.T, ts * 4)
        t0 = time.perf_counter()
        oracle_step(sub(ts), wl.k, wl.backward, router, lo)
        dt = time.perf_counter() - t0
    return sub(ts), ts, es, lo


def sample_desc(wl, ts, es):
    return (f"first {ts} of {wl.T} tokens routed over the first {es} of {wl.E} experts (logits and weights cut "
            f"to them), {'fwd+bwd' if wl.backward else 'fwd'} in float64")


def step_flops(wl, lora_r=0):
    """Useful flops of one step. With adapters of rank r the base weights
    are frozen: the backward has the dgrad GEMMs (6 H I per pair) but no base
    weight gradients, and every adapter product counts (2 r (6H + 9I) per
    pair over the forward and backward)."""
    if lora_r:
        P, H, I = wl.P, wl.H, wl.I
        base = 6.0 * H * I * P * (2 if wl.backward else 1)
        return base + 2.0 * P * lora_r * ((6 * H + 9 * I) if wl.backward else (2 * H + 3 * I))
    return wl.flops_fwd() + (wl.flops_bwd() if wl.backward else 0.0)


def lora_np(wl, args):
    """The bench's adapters as float64 arrays for the oracle."""
    d = lora_inputs(wl, args.lora, args.seed)
    out = {n: d[n].double().numpy() for n in ("A_gu", "B_gu", "A_d", "B_d")}
    out["scale"] = d["scale"]
    return out


def lora_inputs(wl, r, seed, scale=2.0):
    """Seeded rank-r adapters for the workload (bf16; scale = alpha / r)."""
    from routed_grouped_gemm_router_b200.inputs import make_lora
    d = make_lora(wl.E, wl.H, wl.I, r, seed=seed + 1000)
    d["scale"] = scale
    return d


def world_info():
    """(world size, rank, local rank) from the torch.distributed.run environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(values, device):
    """Element-wise max of per-rank values (device-timed milliseconds)."""
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate_tflops(world, flops_per_step, steps, total_ms):
    """Whole-job throughput: every rank processed `steps` steps of its own batch."""
    return world * flops_per_step * steps / (total_ms * 1e-3) / 1e12


def run_reference(args, wl, rank):
    """The oracle timed on the host cores (rank 0 only)."""
    if rank != 0:
        return
    inp = make_inputs(wl, seed=args.seed)
    lo = lora_np(wl, args) if args.lora else None
    sample, ts, es, lo = cpu_sample(inp, wl, target_s=args.ref_step_s, router=args.router_linear, lora=lo)
    sub_wl = type(wl)(wl.name, ts, wl.H, es, wl.k, wl.I, wl.zipf_s, wl.dead_experts, wl.backward)
    for _ in range(args.warmup):
        oracle_step(sample, wl.k, wl.backward, args.router_linear, lo)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(sample, wl.k, wl.backward, args.router_linear, lo)
    dt = (time.perf_counter() - t0) / args.steps
    value = step_flops(sub_wl, args.lora) / dt / 1e12
    desc = sample_desc(wl, ts, es)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, args),
        "tokens_per_s": ts / dt,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def front_end_timing(B, logits, wl, bufs, dev, calls=20, reps=10):
    """Microseconds per call of the routing front end: `calls` calls captured
    in one CUDA graph (so the graph's own launch cost is shared), the graph
    replayed `reps` times; median of three alternating rounds."""
    perm = {n: bufs["perm"][n] for n in ("counts", "offsets", "sorted_pair", "pair_pos")}
    idx, w, probs = bufs["topk_idx"], bufs["topk_w"], bufs["probs"]

    def fused():
        B.moe_route_permute(logits, wl.k, None, idx, w, probs, out=perm, ws=bufs["route_perm_ws"])

    def two_calls():
        B.moe_route(logits, wl.k, idx, w, probs)
        B.moe_permute(idx, wl.E, None, out=perm, ws=bufs["perm_ws"])

    graphs = {}
    side = torch.cuda.Stream()
    for name, fn in (("route_permute_us", fused), ("route_then_permute_us", two_calls)):
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(calls):
                fn()
        graphs[name] = g
    times = {name: [] for name in graphs}
    for _ in range(3):
        for name, g in graphs.items():
            g.replay()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(reps):
                g.replay()
            b.record()
            torch.cuda.synchronize()
            times[name].append(a.elapsed_time(b) * 1e3 / (reps * calls))
    out = {name: sorted(v)[1] for name, v in times.items()}
    del graphs
    out["note"] = (f"ids to permutation without the row gather; {calls} calls per CUDA graph, {reps} replays, "
                   "median of 3 alternating rounds; fused: moe_route_permute (2 kernels), two calls: moe_route + "
                   "moe_permute (4 kernels)")
    return out


def profile_ranges(B, layer, wl, X, logits, dY, W_gu, W_d, bufs):
    """One layer step whose expert-GEMM call (moe_experts_fwd: gate/up then
    down, each a one-CTA tail launch and a pair launch running side by side)
    and whose backward call (moe_layer_bwd) each sit inside a profiler
    start/stop range, for ncu's range replay: the DRAM bytes of a range are
    those of its launches as they ran, concurrently."""
    import torch.cuda.profiler as cuprof
    b = bufs
    idx, w, probs, perm = B.moe_route_permute(logits, wl.k, X, b["topk_idx"], b["topk_w"], b["probs"],
                                              out=b["perm"], ws=b["route_perm_ws"])
    torch.cuda.synchronize()
    cuprof.start()
    h, gu, O = B.moe_experts_fwd(perm["Xp"], perm["offsets"], perm["sorted_pair"], w, wl.T, wl.E, wl.k, W_gu, W_d,
                                 h=b["h"], gu_save=b["gu"], O=b["O"], save_gu=True)
    torch.cuda.synchronize()
    cuprof.stop()
    Y = B.moe_combine(O, perm["pair_pos"], wl.T, wl.k, Y=b["Y"])
    st = layer.LayerState(wl.T, wl.E, wl.k, idx, w, probs, perm, h, gu, O, Y)
    torch.cuda.synchronize()
    cuprof.start()
    layer.backward(st, dY, W_gu, W_d, bufs=b)
    torch.cuda.synchronize()
    cuprof.stop()
    status = B.last_device_status()
    print(json.dumps({"profile_ranges": ["moe_experts_fwd", "moe_layer_bwd"], "workload": wl.name,
                      "device_status": status}), flush=True)
    if status != 0:
        raise RuntimeError(f"device status {B.status_str(status)}")


def workload_config(wl, args):
    return {"workload": f"{wl.name} MoE layer {'fwd+bwd' if wl.backward else 'fwd'}: T={wl.T} H={wl.H} "
                        f"E={wl.E} k={wl.k} I={wl.I}" + (f" zipf_s={wl.zipf_s}" if wl.zipf_s else "")
                        + (" + router Linear (fp32, on the GPU)" if getattr(args, "router_linear", False) else "")
                        + (f" + LoRA rank {args.lora} on the expert weights (base frozen)"
                           if getattr(args, "lora", 0) else ""),
            "router_linear": bool(getattr(args, "router_linear", False)),
            "gather_fused": bool(getattr(args, "gather_fused", False)),
            "cuda_graph": bool(getattr(args, "cuda_graph", False)),
            "dw_dtype": "f32" if getattr(args, "dw_f32", False) else "bf16",
            "lora_rank": int(getattr(args, "lora", 0)),
            "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k, "I": wl.I, "seed": args.seed,
            "l2": "flushed between timed steps (256 MiB write outside the timed events)",
            "parallelism": (f"ep{args.gpus} (own batch per rank, E/{args.gpus} experts per rank, rows to their "
                            "owners and back by all-to-all over NCCL)" if getattr(args, "ep", False) else
                            f"dp{args.gpus} (own batch per rank, weight gradients summed over NCCL: "
                            f"{getattr(args, 'grad_sync', 'allreduce')})" if args.gpus > 1 and wl.backward
                            and getattr(args, "grad_sync", "allreduce") != "none"
                            else f"replicas x{args.gpus}" if args.gpus > 1 else "single GPU")}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="qwen3-235b-a22b", choices=sorted(WORKLOADS))
    ap.add_argument("--forward-only", action="store_true")
    ap.add_argument("--cuda-graph", action="store_true",
                    help="capture one whole step in a CUDA graph after warm-up and time its replays")
    ap.add_argument("--gather-fused", action="store_true",
                    help="GEMMs read X / dY rows by token (no Xp / dYp copies) instead of the permuted copies")
    ap.add_argument("--lora", type=int, default=0, metavar="R",
                    help="LoRA adapters of rank R on the expert weights; base weights frozen (no dW GEMMs)")
    ap.add_argument("--dw-f32", action="store_true",
                    help="weight gradients written as fp32 (the wgrad accumulators unrounded) instead of bf16")
    ap.add_argument("--router-linear", action="store_true",
                    help="include the router Linear (logits = X W_r^T and its backward) in the step")
    ap.add_argument("--grad-sync", default="allreduce", choices=["allreduce", "reduce_scatter", "none"],
                    help="N > 1: how the ranks' weight gradients are summed after each backward (NCCL)")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallel: each rank owns E/N experts, rows travel to their owners and back "
                         "(all-to-all over NCCL); with one GPU a one-rank group")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-front-end", action="store_true", help="skip the routing front-end graph timing")
    ap.add_argument("--profile-range", action="store_true",
                    help="after warm-up, run one step with the expert-GEMM call and the backward call inside "
                         "profiler start/stop ranges (for ncu range replay), then exit")
    ap.add_argument("--tokens", type=int, default=None, help="override T (smaller profiling cases)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E (scaled profiling cases: fewer experts, the same rows per expert with --tokens)")
    ap.add_argument("--sustained-s", type=float, default=2.0,
                    help="length of the back-to-back sustained pass reported beside the headline (0: skip)")
    ap.add_argument("--cpu-target-s", type=float, default=15.0)
    ap.add_argument("--ref-step-s", type=float, default=4.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = WORKLOADS[args.workload]
    if args.forward_only or args.tokens or args.experts:
        T = args.tokens or wl.T
        E = args.experts or wl.E
        if E < wl.k:
            ap.error("--experts must be at least the workload's top-k")
        name = wl.name + (f"-e{E}" if E != wl.E else "") + (f"-t{T}" if T != wl.T else "")
        wl = type(wl)(name, T, wl.H, E, wl.k, wl.I, wl.zipf_s, min(wl.dead_experts, E - wl.k),
                      wl.backward and not args.forward_only)

    world, rank, local_rank = world_info()
    if args.impl == "reference":
        run_reference(args, wl, rank)
        return

    import torch.distributed as dist
    from routed_grouped_gemm_router_b200 import binding as B
    from routed_grouped_gemm_router_b200 import layer

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    ep_mode = args.ep
    if ep_mode and (args.router_linear or args.lora or args.gather_fused or args.dw_f32 or args.cuda_graph
                    or not wl.backward):
        ap.error("--ep runs the default layer forward + backward, eagerly")
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    elif ep_mode:  # one rank: the exchange is the rank's copy to itself
        import socket
        with socket.socket() as so:
            so.bind(("127.0.0.1", 0))
            port = so.getsockname()[1]
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", str(port))
        dist.init_process_group("nccl", rank=0, world_size=1, device_id=dev,
                                timeout=datetime.timedelta(seconds=120))

    # every rank its own batch: seed + rank
    inp = make_inputs(wl, seed=args.seed + rank, with_dy=wl.backward)
    if ep_mode:
        # expert parallel: this rank holds only its block of experts
        from routed_grouped_gemm_router_b200 import ep as EP
        e_lo, e_hi = EP.experts_of_rank(wl.E, world, rank)
        X, W_gu, W_d = inp.X.to(dev), inp.W_gu[e_lo:e_hi].to(dev), inp.W_d[e_lo:e_hi].to(dev)
    else:
        X, W_gu, W_d = inp.X.to(dev), inp.W_gu.to(dev), inp.W_d.to(dev)
    logits = inp.logits.to(dev)
    W_r = inp.W_r.to(dev)
    dY = inp.dY.to(dev) if wl.backward else None
    rl = args.router_linear
    if rl and wl.zipf_s:
        ap.error("--router-linear: the stress workloads' logit bias has no router-weight form")
    gf = args.gather_fused
    lr = args.lora
    if lr and (rl or gf or args.dw_f32):
        ap.error("--lora runs the permuted-operand layer on the caller's logits with frozen base weights")
    lora = None
    if lr:
        lora = {n: (t.to(dev) if torch.is_tensor(t) else t) for n, t in lora_inputs(wl, lr, args.seed).items()}
    bufs = layer.allocate(wl.T, wl.E, wl.k, wl.H, wl.I, dev, save_gu=True, router=rl, gather=gf,
                          dw_f32=args.dw_f32, lora_r=lr)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    # Data parallel (N > 1): the weight gradients live in one flat buffer and
    # are summed over the ranks after every backward (one NCCL collective),
    # timed on its own with events around it.
    grad_flat, grad_extra, sync_evs = None, [], []
    sync = world > 1 and wl.backward and args.grad_sync != "none" and not ep_mode
    if sync and args.cuda_graph:
        ap.error("--cuda-graph captures one rank's step; the N > 1 step with its gradient exchange runs eagerly")
    if sync:
        from routed_grouped_gemm_router_b200 import dp
        g = bufs["grads"]
        names = [n for n in ("dW_gu", "dW_d", "dA_gu", "dB_gu", "dA_d", "dB_d") if n in g]
        grad_flat, views = dp.flat_views({n: tuple(g[n].shape) for n in names}, g[names[0]].dtype, dev)
        g.update(views)
        if rl:
            grad_extra = [bufs["dW_r"]]

    def exchange():
        """Sums the weight gradients over the ranks (N > 1)."""
        if not sync:
            return
        if torch.cuda.is_current_stream_capturing():
            dp.sync_weight_grads(grad_flat, extra=grad_extra, op=args.grad_sync)
            return
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        dp.sync_weight_grads(grad_flat, extra=grad_extra, op=args.grad_sync)
        b.record(stream)
        sync_evs.append((a, b))

    def run_fwd(X_, logits_, b):
        """The layer's forward through the public API."""
        if ep_mode:
            return EP.ep_forward(logits_, X_, W_gu, W_d, wl.k, wl.E)
        if rl:
            return layer.forward_from_x(X_, W_r, W_gu, W_d, wl.k, bufs=b, gather=gf)
        if lr:
            return layer.forward_lora(logits_, X_, W_gu, W_d, wl.k, lora, bufs=b)
        return layer.forward(logits_, X_, W_gu, W_d, wl.k, bufs=b, gather=gf)

    def run_bwd(st, dY_, X_, b):
        """The layer's backward through the public API."""
        if ep_mode:
            return EP.ep_backward(st, dY_, W_gu, W_d)
        if rl:
            return layer.backward_to_x(st, dY_, X_, W_r, W_gu, W_d, bufs=b)
        if lr:
            return layer.backward_lora(st, dY_, W_gu, W_d, bufs=b)
        return layer.backward(st, dY_, W_gu, W_d, bufs=b)

    def run_step(X_, logits_, dY_, b):
        """One forward (+ backward and, with N > 1, the weight-gradient
        exchange) through the public API; (state, grads)."""
        st = run_fwd(X_, logits_, b)
        g = None
        if wl.backward:
            g = run_bwd(st, dY_, X_, b)
            exchange()
        return st, g

    def step():
        run_step(X, logits, dY, bufs)

    for i in range(args.warmup):
        if i == args.warmup - 1:
            B.profile_enable(True)  # the last warm-up step names the dominant kernel
        step()
    torch.cuda.synchronize()
    warm = B.profile_read()
    B.profile_enable(False)
    warm_dominant = max(warm.items(), key=lambda kv: kv[1][0])[0]
    status = B.last_device_status()
    if status != 0:
        raise RuntimeError(f"device status after warm-up: {B.status_str(status)}")
    # experts that received rows: whose weights the row-grouped GEMMs read
    active, routing = None, None
    if not ep_mode and bufs.get("perm") is not None:
        active = int((bufs["perm"]["counts"] > 0).sum().item())
        routing = routing_stats(bufs["perm"]["counts"].cpu().tolist())

    if args.profile_range:
        if rl or lr or gf or world > 1 or ep_mode:
            ap.error("--profile-range profiles the default layer on one GPU")
        profile_ranges(B, layer, wl, X, logits, dY, W_gu, W_d, bufs)
        return

    graph = None
    if args.cuda_graph:
        # one whole step captured once (profiling off), replayed in the timed pass
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        n0 = B.launch_count()
        with torch.cuda.graph(graph):
            step()
        graph_launches = B.launch_count() - n0  # the library's kernels in one captured step
        torch.cuda.synchronize()
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize()

    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
    def timed_steps(only=None, profile=True, replay=False, nsteps=None):
        """K (or nsteps) steps, each bracketed by events on the launching
        stream, L2 flushed between steps outside the events; the library also
        records CUDA events around its kernel launches (all of them, or only
        kernel `only`)."""
        nsteps = nsteps or args.steps
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(nsteps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        if profile:
            B.profile_enable(True)
            if only is not None:
                B.profile_only(only)
        for i in range(nsteps):
            flush.zero_()
            evs[i][0].record(stream)
            if replay:
                graph.replay()
            else:
                step()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        prof = None
        if profile:
            prof = B.profile_read()
            # effective SM clock of each GEMM, from the kernels' own cycle and
            # nanosecond counters (NVML's clock reading does not resolve them)
            for n in list(prof):
                if n.startswith("gemm_"):
                    prof[n] = prof[n] + (B.profile_read_clock(n),)
            B.profile_enable(False)
        status = B.last_device_status()
        if status != 0:
            raise RuntimeError(f"device status after timed steps: {B.status_str(status)}")
        return [a.elapsed_time(b) for a, b in evs], prof

    # Pass 1 is the headline: the step time right after warm-up, with events
    # around the GEMM that dominated the warm-up steps only. Pass 2 records
    # every kernel (per-kernel table; event records between launches
    # serialise them, and under sustained tensor load the power limit lowers
    # the clock after some 50 ms, so pass 2 runs slower).
    # With --cuda-graph the headline pass replays the captured step (no
    # library events inside it) and the dominant kernel is timed in an extra
    # eager pass right after.
    dom = warm_dominant
    sync_evs.clear()
    if sampler:
        sampler.window(True)
    n_launch0 = B.launch_count()
    if graph is not None:
        step_ms, _ = timed_steps(profile=False, replay=True)
        head_launches = graph_launches * args.steps
    else:
        step_ms, dom_prof = timed_steps(only=dom)
        head_launches = B.launch_count() - n_launch0  # the library's kernels inside the headline pass
    if sampler:
        sampler.window(False)
    torch.cuda.synchronize()
    sync_ms = sum(a.elapsed_time(b) for a, b in sync_evs)  # the exchange inside the headline steps
    if graph is not None:
        _, dom_prof = timed_steps(only=dom)
    total_ms = sum(step_ms)
    prof_step_ms, prof = timed_steps()
    # Pass 3, sustained: the same steps back to back for about --sustained-s
    # seconds with no library events (a training run's steady state under the
    # power limit), reported beside the headline.
    sus_ms = None
    if args.sustained_s > 0:
        n_sus = max(args.steps, int(args.sustained_s * 1e3 / (total_ms / args.steps)) + 1)
        if world > 1:  # every rank runs the same number of steps
            n_sus = int(max_over_ranks([n_sus], dev)[0])
        sus_ms, _ = timed_steps(profile=False, replay=graph is not None, nsteps=n_sus)

    # Routing front end alone (ids -> permutation, no row gather), replayed
    # from CUDA graphs back to back: the fused call (routing with the expert
    # counts, then one scan-and-scatter kernel) and the two-call path
    # (moe_route, then moe_permute's count, scan and scatter kernels).
    front = None
    if not args.no_front_end and rank == 0 and not rl:
        front = front_end_timing(B, logits, wl, bufs, dev)

    # End to end through the public API with host buffers: every step copies
    # its inputs (X, logits, dY) from pinned host memory and reads its results
    # (Y, dX, dlogits) back. Inputs and outputs are double-buffered and the
    # copies run on two copy streams, so step i+1's upload and step i's
    # download overlap step i's compute, as a training loop would prefetch:
    # the forward starts once X and the logits are in (dY lands meanwhile),
    # and Y goes back while the backward runs.
    e2e_ms, h2d, d2h = None, 0, 0
    if not args.no_e2e:
        pin = dict(X=inp.X.pin_memory(), logits=inp.logits.pin_memory(),
                   dY=inp.dY.pin_memory() if wl.backward else None)
        out_h = dict(Y=torch.empty(wl.T, wl.H, dtype=torch.bfloat16).pin_memory(),
                     dX=torch.empty(wl.T, wl.H, dtype=torch.bfloat16).pin_memory(),
                     dlogits=torch.empty(wl.T, wl.E, dtype=torch.float32).pin_memory())
        h2d = (pin["X"].numel() * 2 + (0 if rl else pin["logits"].numel() * 4)
               + (pin["dY"].numel() * 2 if wl.backward else 0))
        d2h = out_h["Y"].numel() * 2 + ((out_h["dX"].numel() * 2 + out_h["dlogits"].numel() * 4)
                                        if wl.backward else 0)
        din = [dict(X=torch.empty_like(X), logits=torch.empty_like(logits),
                    dY=torch.empty_like(dY) if wl.backward else None) for _ in range(2)]
        obufs = []
        for _ in range(2):
            o = dict(bufs)
            o["Y"] = torch.empty_like(bufs["Y"])
            o["grads"] = dict(bufs["grads"])
            o["grads"]["dX"] = torch.empty_like(bufs["grads"]["dX"])
            o["grads"]["dlogits"] = torch.empty_like(bufs["grads"]["dlogits"])
            obufs.append(o)
        up, down = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        ev_in_f, ev_in_b, ev_used = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        ev_y, ev_out, ev_copied = [ev(), ev()], [ev(), ev()], [ev(), ev()]

        def upload(b):
            with torch.cuda.stream(up):
                up.wait_event(ev_used[b])
                din[b]["X"].copy_(pin["X"], non_blocking=True)
                if not rl:
                    din[b]["logits"].copy_(pin["logits"], non_blocking=True)
                ev_in_f[b].record(up)  # what the forward reads
                if wl.backward:
                    din[b]["dY"].copy_(pin["dY"], non_blocking=True)
                ev_in_b[b].record(up)

        def run_e2e(nsteps):
            for b in range(2):
                ev_used[b].record(stream)
                ev_copied[b].record(stream)
            upload(0)
            for i in range(nsteps):
                b = i % 2
                if i + 1 < nsteps:
                    upload((i + 1) % 2)
                stream.wait_event(ev_in_f[b])
                stream.wait_event(ev_copied[b])  # this buffer's previous results are home
                st = run_fwd(din[b]["X"], din[b]["logits"], obufs[b])
                ev_y[b].record(stream)
                with torch.cuda.stream(down):
                    down.wait_event(ev_y[b])
                    out_h["Y"].copy_(st.Y, non_blocking=True)
                g = None
                if wl.backward:
                    stream.wait_event(ev_in_b[b])
                    g = run_bwd(st, din[b]["dY"], din[b]["X"], obufs[b])
                    exchange()
                ev_used[b].record(stream)
                ev_out[b].record(stream)
                with torch.cuda.stream(down):
                    down.wait_event(ev_out[b])
                    if wl.backward:
                        out_h["dX"].copy_(g["dX"], non_blocking=True)
                        out_h["dlogits"].copy_(g["dlogits"], non_blocking=True)
                    ev_copied[b].record(down)
            stream.wait_event(ev_copied[(nsteps - 1) % 2])

        run_e2e(args.warmup)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        run_e2e(args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e2e_ms = e0.elapsed_time(e1)
    clocks = sampler.stop() if sampler else None

    sus_total = sum(sus_ms) if sus_ms else None
    if world > 1:
        t_max, e_max, s_max, sync_ms = max_over_ranks([total_ms, e2e_ms or 0.0, sus_total or 0.0, sync_ms], dev)
        total_ms, e2e_ms = t_max, (e_max if e2e_ms is not None else None)
        sus_total = s_max if sus_ms else None
    if rank != 0:
        if dist.is_initialized():
            dist.destroy_process_group()
        return

    flops = step_flops(wl, lr)
    ms_per_step = total_ms / args.steps
    value = aggregate_tflops(world, flops, args.steps, total_ms)
    e2e_value = aggregate_tflops(world, flops, args.steps, e2e_ms) if e2e_ms else None
    peaks, peaks_src = read_peaks()

    # dominant kernel: most device time over the timed region
    kernels = {}
    for name, rec in prof.items():
        ms, n = rec[0], rec[1]
        kind, work = kernel_work(name, wl, lr, peaks, active)
        avg_ms = ms / n
        rate = work / (avg_ms * 1e-3)
        kernels[name] = {"ms_per_step": ms / args.steps, "launches": n, "share": ms / sum(prof_step_ms),
                         "bound": kind,
                         "achieved": rate / 1e12 if kind == "tensor" else rate / 1e9,
                         "unit": "TFLOP/s" if kind == "tensor" else "GB/s"}
        if len(rec) > 2:
            kernels[name]["sm_mhz_in_kernel"] = round(rec[2])
    kind, work = kernel_work(dom, wl, lr, peaks, active)
    avg_s = dom_prof[dom][0] / dom_prof[dom][1] * 1e-3
    if kind == "tensor":
        achieved = work / avg_s / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_sustained": peaks["bf16_tflops_sustained"],
                "frac_sustained": achieved / peaks["bf16_tflops_sustained"]}
    else:
        achieved = work / avg_s / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak}
    if len(dom_prof[dom]) > 2:
        roof["sm_mhz_in_kernel"] = round(dom_prof[dom][2])
        if clocks is not None:
            # NVML's reading is a coarse average: the kernel's own counters
            # give the clock it really ran at in the headline pass
            clocks["dominant_gemm_sm_mhz_in_kernel"] = round(dom_prof[dom][2])
            clocks["note"] = ("in-kernel SM clock = the dominant GEMM's own clock64 cycles / globaltimer ns over its "
                              "main loops; it sits below NVML's reading because the 1000 W power limit slows the "
                              "clock inside the tensor-bound kernels, which NVML's coarse sampling does not resolve "
                              "(the cuBLAS sustained peak in MEASURED_PEAKS.json was taken at a 1327 MHz median with "
                              "no throttle reason flagged either); no clock lock is set")
    # the committed captures are of the default layer: LoRA, fp32 weight
    # gradients and gathered operands change what the GEMMs move
    same_kernels = not (lr or args.dw_f32 or gf)
    traffic, traffic_src = measured_traffic(dom, wl.name) if same_kernels else (None, None)
    roof["peak_datasheet"], roof["frac_datasheet"] = datasheet_fracs(roof)
    roof.update({"kernel": dom, "traffic": traffic, "traffic_source": traffic_src,
                 "algorithmic_per_launch": work, "experts_with_rows": active,
                 "peak_source": f"{peaks_src} (MEASURED_PEAKS.json)" if peaks_src == "measured" else "fallback"})

    cpu = None
    if not args.no_cpu_baseline and world == 1:  # the oracle baseline is timed at N = 1 only
        lo = lora_np(wl, args) if lr else None
        sample, ts, es, lo = cpu_sample(inp, wl, target_s=args.cpu_target_s, router=rl, lora=lo)
        t0 = time.perf_counter()
        oracle_step(sample, wl.k, wl.backward, args.router_linear, lo)
        dt = time.perf_counter() - t0
        sub_wl = type(wl)(wl.name, ts, wl.H, es, wl.k, wl.I, wl.zipf_s, wl.dead_experts, wl.backward)
        cpu = {"value": step_flops(sub_wl, lr) / dt / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": sample_desc(wl, ts, es) + f", one run of {dt:.1f} s"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights)",
        "config": workload_config(wl, args),
        "tokens_per_s": world * wl.T * args.steps / (total_ms * 1e-3),
        "pct_of_bf16_peak": value / world / peaks["bf16_tflops"],
        "pct_of_bf16_peak_datasheet": value / world / DATASHEET_PEAKS["bf16_tflops"],
        "roofline": roof, "cpu_baseline": cpu,
        "e2e": None if e2e_ms is None else {
            "value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": e2e_ms / args.steps,
            "note": "pinned host buffers; uploads/downloads on two copy streams overlap compute (the forward "
                    "starts once X and the logits are in, Y goes back during the backward); no L2 flush "
                    "(per-step working set >> L2)"},
        "routing": routing,
        "gpu_launches": head_launches, "clocks": clocks, "kernels": kernels, "front_end": front,
        "kernels_note": "value, ms_per_step and the roofline kernel come from the first timed pass (events "
                        "around the dominant kernel only); the per-kernel table from a second pass that records "
                        "every launch (serialised, and later under the power limit)",
        "ms_per_step_profiled": sum(prof_step_ms) / args.steps,
        "grad_sync": None if not sync else {
            "op": args.grad_sync, "backend": "nccl",
            "bytes_per_step": grad_flat.numel() * grad_flat.element_size() + sum(t.numel() * t.element_size()
                                                                                  for t in grad_extra),
            "ms_per_step": sync_ms / args.steps,
            "note": "sum of the ranks' weight gradients after each backward, inside the timed step; events "
                    "around the collective in the headline pass, max over ranks"},
        "sustained": None if not sus_ms else {
            "value": aggregate_tflops(world, flops, len(sus_ms), sus_total), "unit": UNIT,
            "ms_per_step": sus_total / len(sus_ms), "steps": len(sus_ms), "seconds": sus_total * 1e-3,
            "pct_of_bf16_peak_sustained": aggregate_tflops(world, flops, len(sus_ms), sus_total) / world
            / peaks["bf16_tflops_sustained"],
            "note": "the same steps back to back after the per-kernel pass, no library events; L2 flushed "
                    "between steps outside the events"},
    }
    print(json.dumps(line), flush=True)
    if dist.is_initialized():
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
